"""The host n-gram drafter feeding the one-hot verification path end to end.

A synthetic rollout history (each rollout of a prompt repeats the previous
one with 10% of its tokens replaced) fills NgramDrafter; one call of
draft_batch drafts for a whole batch of positions in new rollouts, straight
into draft_tokens / draft_lens, and spec_verify (no draft logits) verifies
them against target rows whose favoured token is the rollout's true next
token (NgramRL essay "AI 开始抄自己的作业——而且抄得理直气壮", sections
"📓 NgramRL：每道题配一本活页草稿本" and "⚡ 投机解码：让草稿先跑，考官殿后").

* sampling: the GPU outcome equals the oracle's on the same inputs;
* greedy: each request accepts exactly the drafts that match the true
  continuation up to the first mismatch (argmax = the favoured token).
"""
import numpy as np
import pytest

from speculative_decoding_verification_92_b200 import host
from speculative_decoding_verification_92_b200.workload import F32, make_workload
from helpers import compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def test_batched_ngram_drafts_feed_one_hot_verification():
    rng = np.random.default_rng(77)
    P, T, V, B, k = 12, 240, 4096, 48, 8
    rollout = [rng.integers(0, V, T).astype(np.int32) for _ in range(P)]

    def vary(r):
        r = r.copy()
        m = rng.random(T) < 0.1
        r[m] = rng.integers(0, V, int(m.sum()))
        return r

    ng = host.NgramDrafter(6, 4)
    for _ in range(3):
        ng.begin_step()
        for p in range(P):
            rollout[p] = vary(rollout[p])
            ng.add(p, rollout[p])
    new = [vary(r) for r in rollout]
    pids = rng.integers(0, P, B)
    pos = rng.integers(8, T - k - 1, B)
    tok, lens = ng.draft_batch(pids, [new[p][:q] for p, q in zip(pids, pos)], k)
    truth = np.stack([new[p][q:q + k + 1] for p, q in zip(pids, pos)])
    assert lens.min() >= 0 and (lens == k).mean() > 0.5

    w = make_workload(B=B, k_max=k, V=V, dtype=F32, seed=78, z_sigma=1.0, boost=0.0, draft_mode="ids",
                      lens=lens)
    w.tokens[:] = tok
    for b in range(B):
        for i in range(int(lens[b]) + 1):
            w.target[b, i, truth[b, i]] += np.float32(10.0)

    o = run_oracle(w, diag=True)
    g_len, g_tok = run_gpu(w)
    compare(w, g_len, g_tok, o, diag=o)

    og = run_oracle(w, greedy=True)
    gg_len, gg_tok = run_gpu(w, greedy=True)
    compare(w, gg_len, gg_tok, og, greedy=True)
    match = np.array([next((i for i in range(int(lens[b])) if tok[b, i] != truth[b, i]), int(lens[b]))
                      for b in range(B)])
    assert np.array_equal(gg_len, match)
    assert np.array_equal(gg_tok[np.arange(B), gg_len], truth[np.arange(B), match])
