"""Pins of the CPU oracle to facts outside the oracle itself.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises
``AssertionError`` when the oracle disagrees with what the pages or the
mathematics fix:

* the worked example printed on the NgramRL essay ("AI 开始抄自己的作业——而且抄得
  理直气壮", section "⚡ 投机解码：让草稿先跑，考官殿后"), stored in
  ``tests/golden/worked_example.json``;
* closed forms of the log-sum-exp and of the rule (q == p always accepts, a
  zero-probability draft always rejects, a one-hot draft's residual is p with
  the drafted token removed);
* library routines (``scipy.special.logsumexp`` / ``softmax``,
  ``numpy.searchsorted``) on special cases that reduce to them;
* the losslessness invariant of the same page and of its section
  "👨🏫 考官坐镇：为什么抄作业不算作弊", checked exactly by enumerating drafts and
  measuring the oracle's acceptance / draw regions by bisection, and
  statistically with a chi-square test over 10^6 seeded trials;
* the sequential rule of "今热点：让AI草稿模型学会"照镜子"" (001ce.com), section
  "先搞懂投机解码在干什么": nothing after the first rejection can change the
  outcome.

The same functions run against deliberately broken copies of the oracle in
``test_oracle_mutants.py`` to show that a plausible slip fails at least one.
"""
from __future__ import annotations

import json
import math
from pathlib import Path

import numpy as np
from scipy.special import logsumexp, softmax
from scipy.stats import chi2

GOLDEN = Path(__file__).resolve().parent / "golden"
ONE_MINUS = float(np.nextafter(1.0, 0.0))


def run1(orc, target, draft, tokens, u, T=1.0, greedy=False, lens=None, diag=False):
    """Verify a single request; returns (j, emitted tokens, flags[, diag])."""
    target = np.asarray(target, np.float32)[None]
    k = target.shape[1] - 1
    draft = None if draft is None else np.asarray(draft, np.float32).reshape(1, k, -1)
    tokens = np.asarray(tokens, np.int32).reshape(1, k)
    u = None if u is None else np.asarray(u, np.float64).reshape(1, k + 1)
    lens_arr = None if lens is None else np.asarray([lens], np.int32)
    out = orc.verify(target, draft, tokens, lens_arr, u, T, greedy, diag=diag)
    res = (int(out["len"][0]), out["tokens"][0].copy(), int(out["flags"][0]))
    return res + (out,) if diag else res


def accept_threshold(orc, target, draft, tokens, i, T=1.0, lens=None):
    """a_i measured from the oracle: the infimum of the u_i values it rejects.
    Earlier positions get u = 0 (accepted whenever their a > 0)."""
    k = len(tokens)

    def accepts(ui):
        u = np.zeros(k + 1)
        u[i] = ui
        j, _, _ = run1(orc, target, draft, tokens, u, T, lens=lens)
        assert j >= i, "an earlier position was rejected with u = 0"
        return j > i

    if not accepts(0.0):
        return 0.0
    if accepts(ONE_MINUS):
        return 1.0
    lo, hi = 0.0, ONE_MINUS
    for _ in range(80):
        mid = 0.5 * (lo + hi)
        if mid <= lo or mid >= hi:
            break
        if accepts(mid):
            lo = mid
        else:
            hi = mid
    return hi


def draw_measure(orc, target, draft, tokens, u_fixed, V, T=1.0, lens=None):
    """Probability of each emitted token at position j when only the final
    uniform u* varies over [0, 1), measured by bisection on the oracle's
    (monotone) inverse-CDF map."""
    k = len(tokens)
    j_ref = None

    def tok(us):
        nonlocal j_ref
        u = np.array(u_fixed, np.float64).copy()
        u[k] = us
        j, toks, _ = run1(orc, target, draft, tokens, u, T, lens=lens)
        if j_ref is None:
            j_ref = j
        assert j == j_ref, "accept length changed with the final uniform"
        return int(toks[j])

    probs = np.zeros(V)
    prev = 0.0
    for t in range(V):
        if t == V - 1 or tok(ONE_MINUS) <= t:
            bound = 1.0
        elif tok(0.0) > t:
            bound = 0.0
        else:
            lo, hi = 0.0, ONE_MINUS
            for _ in range(80):
                mid = 0.5 * (lo + hi)
                if mid <= lo or mid >= hi:
                    break
                if tok(mid) > t:
                    hi = mid
                else:
                    lo = mid
            bound = hi
        probs[t] = bound - prev
        prev = max(prev, bound)
    return probs


def sm(z, T=1.0):
    return softmax(np.asarray(z, np.float64) / T)


# --------------------------------------------------------------------------
# Worked example printed on the page.


def pin_worked_example(orc):
    gold = json.loads((GOLDEN / "worked_example.json").read_text())
    for case in gold["cases"]:
        p, q = case["p_at_x"], case["q_at_x"]
        target = [[math.log(p), math.log(1 - p)], [0.0, 0.0]]
        draft = [[math.log(q), math.log(1 - q)]]
        a = accept_threshold(orc, target, draft, [0], 0)
        tol = case.get("accept_probability_printed_precision", 1e-6)
        assert abs(a - case["accept_probability"]) <= tol, (case["name"], a)
        if "redraw_token" in case:
            for us in (0.0, 0.3, 0.9999):
                j, toks, _ = run1(orc, target, draft, [0], [ONE_MINUS, us])
                assert j == 0 and toks[0] == case["redraw_token"], (j, toks)


# --------------------------------------------------------------------------
# Softmax / log-sum-exp closed forms and library routines.


def _lse_of_rows(orc, rows, T):
    rows = np.asarray(rows, np.float32)
    k = rows.shape[0] - 1
    out = orc.verify(rows[None], None, np.zeros((1, k), np.int32), None,
                     np.zeros((1, k + 1)), T, diag=True)
    return out["lse_t"][0]


def pin_lse_closed_forms(orc):
    for T in (1.0, 0.6, 2.5):
        V = 1000
        c = 1.5
        lse = _lse_of_rows(orc, np.full((1, V), c), T)[0]
        want = c / T + math.log(V)
        assert abs(lse - want) <= 1e-12 * abs(want), (T, lse, want)
        # two-valued row: n1 entries a, n2 entries b
        n1, n2, a, b = 7, 993, 3.25, -1.75
        row = np.full(V, b, np.float32)
        row[::143][:n1] = a
        assert (row == a).sum() == n1
        lse = _lse_of_rows(orc, row[None], T)[0]
        want = math.log(n1 * math.exp(a / T) + n2 * math.exp(b / T))
        assert abs(lse - want) <= 1e-12 * abs(want), (T, lse, want)


def pin_lse_matches_scipy(orc):
    rng = np.random.default_rng(7)
    for T in (1.0, 0.6):
        rows = (rng.normal(0, 3, (3, 4099))).astype(np.float32)
        lse = _lse_of_rows(orc, rows, T)
        want = logsumexp(rows.astype(np.float64) / T, axis=1)
        assert np.allclose(lse, want, rtol=1e-12, atol=0), (lse, want)


def pin_bf16_lse(orc):
    """bf16 storage: decode bits exactly, then the same statistics."""
    from speculative_decoding_verification_92_b200.workload import bf16_bits_to_f32, f32_to_bf16_bits
    rng = np.random.default_rng(8)
    vals = rng.normal(0, 2, (2, 3001)).astype(np.float32)
    bits = f32_to_bf16_bits(vals)
    decoded = bf16_bits_to_f32(bits).astype(np.float64)
    out = orc.verify(bits[None], None, np.zeros((1, 1), np.int32), None,
                     np.zeros((1, 2)), 0.8, diag=True)
    want = logsumexp(decoded / 0.8, axis=1)
    assert np.allclose(out["lse_t"][0], want, rtol=1e-12, atol=0)


def pin_shift_invariance(orc):
    rng = np.random.default_rng(9)
    V = 64
    z = (rng.integers(-256, 256, (2, V)) / 64.0).astype(np.float32)   # exact dyadics
    x = [int(np.argmax(z[0]))]
    for shift in (0.0, 8.0, -20.0):
        _, _, _, out = run1(orc, z + np.float32(shift), None, x, [0.5, 0.5], 0.9, diag=True)
        if shift == 0.0:
            p_ref = out["p"][0, 0]
        assert abs(out["p"][0, 0] - p_ref) <= 1e-13, (shift, out["p"][0, 0], p_ref)
    assert abs(p_ref - sm(z[0], 0.9)[x[0]]) <= 1e-13


# --------------------------------------------------------------------------
# Closed forms of the rule.


def pin_identical_draft_always_accepts(orc):
    rng = np.random.default_rng(10)
    V, k = 50, 5
    for T in (1.0, 0.7):
        z = rng.normal(0, 2, (k + 1, V)).astype(np.float32)
        for _ in range(20):
            toks = rng.integers(0, V, k)
            u = rng.random(k + 1)
            u[:k] = np.maximum(u[:k], 0.999999)   # hardest uniforms
            j, _, _ = run1(orc, z, z[:k], toks, u, T)
            assert j == k, j


def pin_zero_probability_draft_rejects(orc):
    V = 10
    z = np.linspace(-1, 1, V).astype(np.float32)
    z[3] = -np.inf
    target = np.stack([z, z])
    # one-hot draft at the impossible token, and a draft row that likes it
    y = np.zeros((1, V), np.float32)
    y[0, 3] = 5.0
    for draft in (None, y):
        for u0 in (0.0, 0.5):
            j, toks, _ = run1(orc, target, draft, [3], [u0, 0.0])
            assert j == 0, (draft is None, u0, j)
            assert toks[0] != 3
    # with p(3) = 0 the one-hot residual is p itself
    r = draw_measure(orc, target, None, [3], [0.0, 0.0], V)
    assert np.allclose(r, sm(z), atol=1e-12), (r, sm(z))


def pin_one_hot_residual(orc):
    rng = np.random.default_rng(11)
    V = 7
    for T in (1.0, 0.5):
        z = rng.normal(0, 1, (2, V)).astype(np.float32)
        p = sm(z[0], T)
        for x in range(V):
            a = accept_threshold(orc, z, None, [x], 0, T)
            assert abs(a - p[x]) <= 1e-14, (a, p[x])
            r = draw_measure(orc, z, None, [x], [ONE_MINUS, 0.0], V, T)
            want = p.copy()
            want[x] = 0.0
            want /= want.sum()
            assert np.allclose(r, want, atol=1e-12), (x, r, want)


def pin_never_draws_zero_weight(orc):
    V = 9
    z = np.linspace(0, 2, V).astype(np.float32)
    z[0] = z[1] = -np.inf
    target = z[None]                 # k = 0: the bonus draw from row 0
    for us in (0.0, 1e-30):
        out = orc.verify(target[None], None, np.zeros((1, 0), np.int32), None,
                         np.array([[us]]), 1.0)
        assert out["tokens"][0, 0] == 2, out["tokens"]


def pin_inverse_cdf_matches_searchsorted(orc):
    rng = np.random.default_rng(12)
    V, n = 50, 4000
    z = rng.normal(0, 1.5, (1, 1, V)).astype(np.float32)
    u = rng.random((n, 1))
    out = orc.verify(z, None, np.zeros((n, 0), np.int32), None, u, 1.0, B=n)
    p = sm(z[0, 0])
    cdf = np.cumsum(p)
    want = np.searchsorted(cdf, u[:, 0] * cdf[-1], side="right")
    # skip draws within 1e-9 of a CDF step (rounding order may differ there)
    gap = np.min(np.abs(u[:, 0:1] * cdf[-1] - cdf[None, :]), axis=1)
    ok = gap > 1e-9
    assert ok.sum() > n * 0.99
    assert np.array_equal(out["tokens"][ok, 0], want[ok])


def pin_lens_zero(orc):
    rng = np.random.default_rng(13)
    V, k = 40, 3
    z = rng.normal(0, 1, (k + 1, V)).astype(np.float32)
    y = rng.normal(0, 1, (k, V)).astype(np.float32)
    for us in (0.05, 0.5, 0.95):
        u = np.array([0.0, 0.0, 0.0, us])
        j, toks, _ = run1(orc, z, y, [1, 2, 3], u, lens=0)
        assert j == 0
        cdf = np.cumsum(sm(z[0]))
        assert toks[0] == np.searchsorted(cdf, us * cdf[-1], side="right")
        assert np.all(toks[1:] == -1)


# --------------------------------------------------------------------------
# Losslessness, exactly (enumeration + bisection) and statistically.


def _enumerate_position(orc, target, draft, prefix, i, V, T, lens=None):
    """Distribution of the token emitted at position i, given that the
    drafts before i (``prefix``) were accepted, summing over the draft's
    choices at i with the oracle's measured a and residual."""
    k = np.asarray(target).shape[0] - 1
    L = k if lens is None else lens
    total = np.zeros(V)
    if i == L:
        toks = list(prefix) + [0] * (k - len(prefix))
        u_fixed = np.zeros(k + 1)
        return draw_measure(orc, target, draft, toks, u_fixed, V, T, lens=lens)
    q = sm(draft[i], T) if draft is not None else None
    choices = range(V)
    for d in choices:
        weight = q[d] if q is not None else None
        toks = list(prefix) + [d] + [0] * (k - len(prefix) - 1)
        a = accept_threshold(orc, target, draft, toks, i, T, lens=lens)
        emitted = np.zeros(V)
        emitted[d] += a
        if a < 1.0:
            u_fixed = np.zeros(k + 1)
            u_fixed[i] = 0.5 * (a + 1.0)
            emitted += (1.0 - a) * draw_measure(orc, target, draft, toks, u_fixed, V, T, lens=lens)
        if weight is None:
            # one-hot drafter: lossless for every fixed drafted id
            assert np.allclose(emitted, sm(target[i], T), atol=1e-12), (i, d, emitted)
        else:
            total += weight * emitted
    return total if q is not None else sm(target[i], T)


def pin_lossless_enumeration(orc):
    rng = np.random.default_rng(14)
    for T in (1.0, 0.7):
        V, k = 5, 2
        z = rng.normal(0, 1.2, (k + 1, V)).astype(np.float32)
        y = (z[:k] + rng.normal(0, 1.0, (k, V))).astype(np.float32)
        p = np.stack([sm(r, T) for r in z])
        # position 0
        got = _enumerate_position(orc, z, y, [], 0, V, T)
        assert np.allclose(got, p[0], atol=1e-12), (got, p[0])
        # position 1 given draft d0 accepted
        d0 = int(np.argmax(sm(y[0], T)))
        got = _enumerate_position(orc, z, y, [d0], 1, V, T)
        assert np.allclose(got, p[1], atol=1e-12), (got, p[1])
        # bonus position k given every draft accepted
        got = _enumerate_position(orc, z, y, [d0, d0], 2, V, T)
        assert np.allclose(got, p[2], atol=1e-12), (got, p[2])
        # draft length 1 inside k_max = 2: the bonus comes from row 1
        got = _enumerate_position(orc, z, y, [d0], 1, V, T, lens=1)
        assert np.allclose(got, p[1], atol=1e-12), (got, p[1])
        # one-hot drafter, V = 6
        V1 = 6
        z1 = rng.normal(0, 1, (2, V1)).astype(np.float32)
        _enumerate_position(orc, z1, None, [], 0, V1, T)


def _chi2_ok(counts, probs):
    n = counts.sum()
    expected = n * probs
    stat = float(((counts - expected) ** 2 / expected).sum())
    return stat, float(chi2.ppf(1 - 1e-6, len(probs) - 1))


def pin_lossless_chi_square(orc, trials=10**6):
    rng = np.random.default_rng(15)
    V, k = 8, 3
    z = rng.normal(0, 1, (k + 1, V)).astype(np.float32)
    y = (z[:k] + rng.normal(0, 0.8, (k, V))).astype(np.float32)
    p = np.stack([sm(r) for r in z])
    q = np.stack([sm(r) for r in y])
    toks = np.stack([rng.choice(V, size=trials, p=q[i]) for i in range(k)], axis=1).astype(np.int32)
    u = rng.random((trials, k + 1))
    out = orc.verify(z[None], y[None], toks, None, u, 1.0, B=trials)
    first = out["tokens"][:, 0]
    stat, bound = _chi2_ok(np.bincount(first, minlength=V), p[0])
    assert stat < bound, ("first token", stat, bound)
    sel = out["len"] >= 1
    stat, bound = _chi2_ok(np.bincount(out["tokens"][sel, 1], minlength=V), p[1])
    assert stat < bound, ("second token | first accepted", stat, bound)
    # one-hot drafter with arbitrary (uniform) drafted ids: still lossless
    toks = rng.integers(0, V, (trials, k)).astype(np.int32)
    out = orc.verify(z[None], None, toks, None, u, 1.0, B=trials)
    stat, bound = _chi2_ok(np.bincount(out["tokens"][:, 0], minlength=V), p[0])
    assert stat < bound, ("one-hot first token", stat, bound)


# --------------------------------------------------------------------------
# Sequential rule, greedy form, invalid input.


def pin_sequential_rule(orc):
    rng = np.random.default_rng(16)
    V, k = 16, 4
    checked = 0
    for _ in range(200):
        z = rng.normal(0, 1, (k + 1, V)).astype(np.float32)
        y = (z[:k] + rng.normal(0, 1.5, (k, V))).astype(np.float32)
        toks = rng.integers(0, V, k)
        u = rng.random(k + 1)
        j, out, _ = run1(orc, z, y, toks, u)
        if j >= k - 1:
            continue
        z2, y2, t2, u2 = z.copy(), y.copy(), toks.copy(), u.copy()
        z2[j + 1:k] = rng.normal(0, 3, (k - 1 - j, V))
        y2[j + 1:] = rng.normal(0, 3, (k - 1 - j, V))
        t2[j + 1:] = rng.integers(0, V, k - 1 - j)
        u2[j + 1:k] = rng.random(k - 1 - j)
        j2, out2, _ = run1(orc, z2, y2, t2, u2)
        assert j2 == j and np.array_equal(out, out2), (j, j2, out, out2)
        checked += 1
    assert checked > 50


def pin_greedy(orc):
    V = 12
    z = np.zeros((3, V), np.float32)
    z[0, [2, 5]] = 4.0          # tie: lowest index wins
    z[1, 7] = 3.0
    z[2, [1, 9]] = 2.0
    j, toks, _ = run1(orc, z, None, [2, 7], None, greedy=True)
    assert j == 2 and list(toks) == [2, 7, 1]
    j, toks, _ = run1(orc, z, None, [5, 7], None, greedy=True)
    assert j == 0 and list(toks) == [2, -1, -1]
    j, toks, _ = run1(orc, z, None, [2, 6], None, greedy=True)
    assert j == 1 and list(toks) == [2, 7, -1]
    j, toks, _ = run1(orc, z, None, [5, 6], None, greedy=True, lens=0)
    assert j == 0 and list(toks) == [2, -1, -1]


def pin_invalid_requests(orc):
    V, k = 10, 3
    z = np.zeros((k + 1, V), np.float32)
    u = np.zeros(k + 1)
    for toks, lens in (([1, 2, 10], None), ([1, -1, 2], None), ([1, 2, 3], 4), ([1, 2, 3], -1)):
        j, out, flags = run1(orc, z, None, toks, u, lens=lens)
        assert j == -1 and np.all(out == -1) and flags & 4, (toks, lens, j, out)
    # ids beyond the request's length are never looked at
    j, out, flags = run1(orc, z, None, [1, -5, 99], u, lens=1)
    assert j >= 0 and not flags & 4


# ---------------------------------------------------------------------------
# acceptance simulation ("今热点：让AI草稿模型学会"照镜子"", sections
# "VAT怎么把"验收规则"塞进训练里" and "第二件事，改权重分配的锚点")

def _sim(orc, p, q, lens=None, u=None, decay=0.8, tokens=None, V=100):
    p = np.asarray(p, np.float64).reshape(1, -1)
    q = np.asarray(q, np.float64).reshape(1, -1)
    k = p.shape[1]
    tokens = np.zeros((1, k), np.int32) if tokens is None else np.asarray(tokens, np.int32).reshape(1, k)
    lens = None if lens is None else np.asarray([lens], np.int32)
    u = None if u is None else np.asarray(u, np.float64).reshape(1, k + 1)
    r = orc.accept_sim(p, q, tokens, lens, u, decay, V=V)
    return {key: (None if v is None else v[0]) for key, v in r.items()}


def pin_accept_sim_closed_forms(orc):
    # the page's worked ratios: q=0.9, pi=0.95 -> 1; q=0.9, pi=0.1 -> 1/9
    r = _sim(orc, [0.95, 0.1], [0.9, 0.9])
    assert r["a"][0] == 1.0 and abs(r["a"][1] - 1.0 / 9.0) < 1e-15
    # constant a = c: E[j] = c (1 - c^L) / (1 - c)
    for c, L in ((0.5, 3), (0.9, 12), (0.25, 1), (0.7, 24)):
        r = _sim(orc, [c] * L, [1.0] * L)
        want = c * (1 - c ** L) / (1 - c)
        assert abs(r["e"] - want) < 1e-12 * max(1.0, want), (c, L, r["e"], want)
    # certain acceptance: E = L; a zero at position 0: E = 0
    assert _sim(orc, [0.3, 0.2, 0.9], [0.1, 0.2, 0.5])["e"] == 3.0
    assert _sim(orc, [0.0, 1.0, 1.0], [0.5, 0.5, 0.5])["e"] == 0.0
    # positions past the length carry NaN, the expectation stops at L
    r = _sim(orc, [0.5, 0.5, 0.5, 0.5], [1.0] * 4, lens=2)
    assert np.isnan(r["a"][2:]).all() and abs(r["e"] - 0.75) < 1e-15


def pin_accept_sim_expectation_by_enumeration(orc):
    """E[j] against the distribution of the first rejection, built by
    enumerating every accept / reject pattern of independent Bernoulli(a_l)."""
    rng = np.random.default_rng(7)
    for L in (1, 2, 5, 9):
        a = rng.uniform(0.05, 1.0, L)
        a[rng.integers(0, L)] = 1.0
        want = 0.0
        for mask in range(1 << L):
            prob, first = 1.0, L
            for l in range(L):
                ok = (mask >> l) & 1
                prob *= a[l] if ok else 1.0 - a[l]
                if not ok and first == L:
                    first = l
            want += prob * first
        r = _sim(orc, a, np.ones(L))
        assert abs(r["e"] - want) < 1e-12, (L, r["e"], want)


def pin_accept_sim_first_rejection_and_weights(orc):
    # the page's example: ten drafts pass, the eleventh is rejected -> the
    # first ten keep full weight, the decay curve starts at the rejection
    L = 16
    p, q = np.full(L, 0.5), np.ones(L)
    u = np.zeros(L + 1)
    u[10] = 0.75                     # 0.75 >= a = 0.5: first rejection at i = 10
    u[11:] = 0.99                    # later uniforms do not matter
    r = _sim(orc, p, q, u=u, decay=0.8)
    assert r["j"] == 10
    assert np.array_equal(r["w"][:11], np.ones(11))
    assert np.allclose(r["w"][11:], 0.8 ** np.arange(1, L - 10), rtol=1e-15, atol=0)
    # the ablation's hard cut-off and a flat curve
    assert np.array_equal(_sim(orc, p, q, u=u, decay=0.0)["w"], np.r_[np.ones(11), np.zeros(L - 11)])
    assert np.array_equal(_sim(orc, p, q, u=u, decay=1.0)["w"], np.ones(L))
    # all accepted: j = L, full weight; padding weight 0
    r = _sim(orc, p, q, lens=5, u=np.zeros(L + 1))
    assert r["j"] == 5 and np.array_equal(r["w"], np.r_[np.ones(5), np.zeros(L - 5)])
    # u == a rejects (accept iff u < a)
    assert _sim(orc, [0.5, 1.0], [1.0, 1.0], u=[0.5, 0.0, 0.0])["j"] == 0
    # invalid requests: -1 and NaN
    r = _sim(orc, [0.5, 0.5], [1.0, 1.0], u=[0, 0, 0], tokens=[1, 100], V=100)
    assert r["j"] == -1 and np.isnan(r["e"]) and np.isnan(r["a"]).all()


def pin_accept_sim_matches_verify_and_monte_carlo(orc):
    """j equals the verification rule's j on the same inputs, and the mean of
    j over independent uniform draws converges to E[j]."""
    rng = np.random.default_rng(11)
    V, k = 12, 6
    z = rng.normal(0, 1.5, (k + 1, V)).astype(np.float32)
    y = (z[:k] + rng.normal(0, 0.8, (k, V))).astype(np.float32)
    toks = [int(np.argmax(y[i] + rng.gumbel(size=V))) for i in range(k)]
    _, _, _, out = run1(orc, z, y, toks, np.zeros(k + 1), diag=True)
    p, q = out["p"][0], out["q"][0]
    js = []
    for _ in range(4000):
        u = rng.random(k + 1)
        j_ver, _, flags = run1(orc, z, y, toks, u)
        r = _sim(orc, p, q, u=u, tokens=toks, V=V)
        if not flags & 1:
            assert r["j"] == j_ver
        js.append(r["j"])
    e = _sim(orc, p, q, tokens=toks, V=V)["e"]
    sd = np.std(js) / math.sqrt(len(js))
    assert abs(np.mean(js) - e) < 5 * sd + 1e-9, (np.mean(js), e, sd)


# --------------------------------------------------------------------------
# Near-tie flags (the oracle flags a request whose |u - min(1, p/q)| at an
# examined position, or whose residual-CDF margin relative to W, is below
# 1e-5) and the two fallback branches of the rule's readings (no step above
# u*W: the largest positive-weight token; zero residual mass: draw from p_j).


def _flags(orc, target, draft, tokens, u, T=1.0):
    j, toks, flags = run1(orc, target, draft, tokens, u, T)
    return j, toks, flags


def pin_accept_tie_band(orc):
    from oracle import FLAG_ACCEPT_TIE
    # a = p(x) = 0.3 for a one-hot draft; a = p/q = 0.3/0.6 = 0.5 with a draft row
    target = [[math.log(0.3), math.log(0.7)], [0.0, 0.0]]
    cases = [(None, 0.3), ([[math.log(0.6), math.log(0.4)]], 0.5)]
    for draft, a in cases:
        for du, flagged in ((5e-6, True), (-5e-6, True), (2e-5, False), (-2e-5, False), (0.3, False)):
            u0 = a + du
            if not 0.0 <= u0 < 1.0:
                continue
            j, _, flags = _flags(orc, target, draft, [0], [u0, 0.5])
            assert bool(flags & FLAG_ACCEPT_TIE) == flagged, (a, du, flags)
            assert j == (1 if u0 < a else 0), (a, du, j)
    # a tie after the first rejection is never examined, so it is not flagged
    target3 = [[math.log(0.3), math.log(0.7)]] * 3
    j, _, flags = _flags(orc, target3, None, [0, 0], [0.9, 0.3, 0.5])
    assert j == 0 and not flags & FLAG_ACCEPT_TIE, (j, flags)


def pin_draw_tie_band(orc):
    from oracle import FLAG_DRAW_TIE
    # bonus draw (k = 0) from p = [1/4, 1/2, 1/4]: CDF steps at 0.25 and 0.75, W = 1
    row = np.log(np.array([1.0, 2.0, 1.0]) / 4.0).astype(np.float32)
    for step, below, above in ((0.25, 0, 1), (0.75, 1, 2)):
        for du, flagged in ((0.5e-5, True), (-0.5e-5, True), (2e-5, False), (-2e-5, False)):
            out = orc.verify(row[None, None], None, np.zeros((1, 0), np.int32), None,
                             np.array([[step + du]]), 1.0)
            flags, tok = int(out["flags"][0]), int(out["tokens"][0, 0])
            assert bool(flags & FLAG_DRAW_TIE) == flagged, (step, du, flags)
            assert tok == (above if du > 0 else below), (step, du, tok)
    # the band is relative to W: a one-hot rejection at x = 1 leaves the
    # residual [1/4, 0, 1/4] (W = 1/2, step at 1/4 in weight, u* = 1/2 there);
    # u* off by 1.5e-5 puts u*W 0.75e-5 from the step: inside an absolute
    # 1e-5 band, outside the relative one (1e-5 W = 0.5e-5)
    target = np.stack([row, row])
    for du, flagged in ((0.5e-5, True), (-0.5e-5, True), (1.5e-5, False), (-1.5e-5, False)):
        j, toks, flags = _flags(orc, target, None, [1], [0.9, 0.5 + du])
        assert j == 0 and toks[0] == (2 if du > 0 else 0), (du, j, toks)
        assert bool(flags & FLAG_DRAW_TIE) == flagged, (du, flags)


def pin_draw_fallback_takes_last_positive_weight(orc):
    from oracle import FLAG_DRAW_FALLBACK
    # p = [1/2, 1/2, 0, 0]; u* = 1 leaves no token t with C_t > u* W, so the
    # rule's fallback applies: the largest t with positive weight (1, not the
    # last index 3 and not the first positive index 0)
    row = np.array([0.0, 0.0, -np.inf, -np.inf], np.float32)
    out = orc.verify(row[None, None], None, np.zeros((1, 0), np.int32), None, np.array([[1.0]]), 1.0)
    assert int(out["tokens"][0, 0]) == 1, out["tokens"]
    assert int(out["flags"][0]) & FLAG_DRAW_FALLBACK
    # away from it the ordinary rule holds and the fallback flag stays clear
    out = orc.verify(row[None, None], None, np.zeros((1, 0), np.int32), None, np.array([[0.25]]), 1.0)
    assert int(out["tokens"][0, 0]) == 0 and not int(out["flags"][0]) & FLAG_DRAW_FALLBACK


def pin_zero_residual_draws_from_p(orc):
    from oracle import FLAG_ZERO_RESIDUAL
    # identical draft: p == q, so a = 1; u_0 = 1 (no uniform in [0, 1) can do
    # it) forces the rejection, the residual max(0, p - q) is all zero, and
    # the draw falls back to p_0 = [1/4, 1/2, 1/4]
    row = np.log(np.array([1.0, 2.0, 1.0]) / 4.0).astype(np.float32)
    target = np.stack([row, row])
    for us, want in ((0.1, 0), (0.6, 1), (0.9, 2)):
        j, toks, flags = _flags(orc, target, row[None], [1], [1.0, us])
        assert j == 0 and toks[0] == want, (us, j, toks)
        assert flags & FLAG_ZERO_RESIDUAL
        # one-hot draft at a token with p = 1: the residual is zero as well
    certain = np.array([[0.0, -np.inf], [0.0, 0.0]], np.float32)
    j, toks, flags = _flags(orc, certain, None, [0], [1.0, 0.7])
    assert j == 0 and toks[0] == 0 and flags & FLAG_ZERO_RESIDUAL, (j, toks, flags)
    # an ordinary rejection never sets the flag
    j, toks, flags = _flags(orc, target, None, [1], [0.9, 0.6])
    assert j == 0 and not flags & FLAG_ZERO_RESIDUAL


ALL_PINS = [
    pin_worked_example,
    pin_lse_closed_forms,
    pin_lse_matches_scipy,
    pin_bf16_lse,
    pin_shift_invariance,
    pin_identical_draft_always_accepts,
    pin_zero_probability_draft_rejects,
    pin_one_hot_residual,
    pin_never_draws_zero_weight,
    pin_inverse_cdf_matches_searchsorted,
    pin_lens_zero,
    pin_accept_tie_band,
    pin_draw_tie_band,
    pin_draw_fallback_takes_last_positive_weight,
    pin_zero_residual_draws_from_p,
    pin_lossless_enumeration,
    pin_lossless_chi_square,
    pin_sequential_rule,
    pin_greedy,
    pin_invalid_requests,
    pin_accept_sim_closed_forms,
    pin_accept_sim_expectation_by_enumeration,
    pin_accept_sim_first_rejection_and_weights,
    pin_accept_sim_matches_verify_and_monte_carlo,
]


if __name__ == "__main__":   # used by the mutant test: run every pin on one library
    import sys
    sys.path.insert(0, str(Path(__file__).resolve().parents[1]))
    from oracle import Oracle
    orc = Oracle(sys.argv[1])
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError as e:
            print(f"CAUGHT by {pin.__name__}: {str(e)[:200]}")
            sys.exit(3)
    print("NOT CAUGHT")
    sys.exit(0)
