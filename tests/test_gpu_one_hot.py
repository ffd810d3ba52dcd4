"""The one-hot (model-free drafter) path at the full vocabulary, V = 151,936,
in the two regimes the n-gram workload's own parameters do not reach.

* Drafts that the target almost always accepts: the n-gram drafter's ids
  are the target's favoured token (k = 16 drafts, as in the NgramRL essay
  "AI 开始抄自己的作业——而且抄得理直气壮", section "📓 NgramRL：每道题配一本活页草稿本"),
  with the favoured logit boosted by +16 so that p(x) is about 0.97.  Most
  steps accept every draft and draw the bonus token from p at row L.
* A rejection where the drafted token holds p(x) > 0.999: the redraw comes
  from p with the drafted token removed, a distribution of total weight
  1 - p(x) < 1e-3 whose largest piece is the drafted id's own piece.  The
  uniform of position 0 is set above p(x), so every request rejects there.

Both compare every request with the oracle (exact, or a legal outcome where
the oracle flags a near tie)."""
import numpy as np
import pytest

from speculative_decoding_verification_92_b200.workload import make_config
from helpers import compare, run_gpu, run_oracle
from oracle import FLAG_ACCEPT_TIE

pytestmark = pytest.mark.gpu


def test_one_hot_drafts_mostly_accepted_at_full_vocabulary():
    w = make_config(3, boost=16.0, fav_prob=1.0)
    g_len, g_tok = run_gpu(w)
    o = run_oracle(w, diag=True)
    counts = compare(w, g_len, g_tok, o, diag=o)
    assert counts["exact"] + counts["tie_ok"] == w.B
    mean_len = float(np.mean(g_len))
    all_accepted = int((g_len == w.k_max).sum())
    print(f"one-hot, boost 16: {counts}, mean accept {mean_len:.2f} of {w.k_max}, all accepted in {all_accepted}")
    assert mean_len > 10.0
    assert all_accepted > w.B // 4          # many bonus draws from row L at V = 151,936


def test_one_hot_rejection_when_the_draft_holds_almost_all_mass():
    w = make_config(3, B=48, boost=23.0, fav_prob=1.0)
    o = run_oracle(w, diag=True)
    p0 = o["p"][:, 0]
    assert p0.min() > 0.999, p0.min()
    # u_0 in (p(x), 1): every request rejects its first draft
    w.uniforms[:, 0] = np.float32(1.0 - 2.0 ** -24)     # the largest float32 below 1
    assert np.all(w.uniforms[:, 0].astype(np.float64) > p0)
    o = run_oracle(w, diag=True)
    assert np.all(o["len"] == 0)
    g_len, g_tok = run_gpu(w)
    counts = compare(w, g_len, g_tok, o, diag=o)
    assert counts["exact"] + counts["tie_ok"] == w.B
    # u_0 can sit within 1e-5 of p(x) (an acceptance tie, either outcome legal)
    rejected = g_len == 0
    assert np.all(rejected | ((o["flags"] & FLAG_ACCEPT_TIE) != 0))
    assert rejected.sum() >= w.B - 4
    # the redraw never returns the drafted token itself
    assert np.all(g_tok[rejected, 0] != w.tokens[rejected, 0])
    print(f"one-hot rejections at p(x) > 0.999: {counts}")
