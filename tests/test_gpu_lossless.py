"""Losslessness of the GPU path, checked against the mathematics rather than
against the oracle.

Speculative sampling is lossless: whatever the draft distribution q, the token
emitted at a position is distributed as the target softmax p at that position
(NgramRL essay "AI 开始抄自己的作业——而且抄得理直气壮", sections "⚡ 投机解码：让草稿先跑，
考官殿后" and "👨🏫 考官坐镇：为什么抄作业不算作弊").  Here one pair of logit rows
is repeated over a million seeded trials, the drafted ids are sampled from q
on the host (drafter behaviour, not the rule), and the tokens the library
emits are binned and held to p by a chi-square test at the 1 - 1e-6 quantile:

* position 0 with draft logits: accepted draft or residual redraw, ~ p_0;
* the bonus token of trials that accepted their draft, ~ p_1;
* the same two with a one-hot drafter (ids from q, passed without logits).

p and q are computed here in float64 from the stored logits, so nothing in
this file comes from the oracle or the CUDA path.
"""
import numpy as np
import pytest
import torch
from scipy import stats

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import bf16_bits_to_f32, f32_to_bf16_bits

pytestmark = pytest.mark.gpu

TRIALS = 1_000_000
PER_CALL = 20_000
T = 0.8
MIN_EXPECTED = 50.0


def softmax64(z):
    x = z.astype(np.float64) / T
    e = np.exp(x - x.max())
    return e / e.sum()


def stored_rows(dtype, V, seed):
    """Target rows 0 and 1 and draft row 0 as stored on the device, and their
    float32 values."""
    rng = np.random.default_rng(seed)
    z = rng.normal(0.0, 2.0, size=(2, V)).astype(np.float32)
    y = (z[0] + rng.normal(0.0, 1.0, size=V)).astype(np.float32)
    if dtype == "bf16":
        zb, yb = f32_to_bf16_bits(z), f32_to_bf16_bits(y)
        return (torch.from_numpy(zb.view(np.int16)).view(torch.bfloat16),
                torch.from_numpy(yb.view(np.int16)).view(torch.bfloat16), bf16_bits_to_f32(zb), bf16_bits_to_f32(yb))
    return torch.from_numpy(z), torch.from_numpy(y), z, y


def chi2_holds(counts, p):
    """Chi-square of observed counts against probabilities p: tokens expected
    at least MIN_EXPECTED times are their own bin, the rest are pooled in
    order of p into bins of at least MIN_EXPECTED."""
    n = counts.sum()
    order = np.argsort(-p, kind="stable")
    obs, exp = [], []
    o_acc = e_acc = 0.0
    for t in order:
        o_acc += counts[t]
        e_acc += n * p[t]
        if e_acc >= MIN_EXPECTED:
            obs.append(o_acc)
            exp.append(e_acc)
            o_acc = e_acc = 0.0
    if e_acc > 0.0:
        obs[-1] += o_acc
        exp[-1] += e_acc
    obs, exp = np.asarray(obs), np.asarray(exp)
    stat = float(((obs - exp) ** 2 / exp).sum())
    bound = float(stats.chi2.ppf(1.0 - 1e-6, len(obs) - 1))
    return stat, bound, len(obs)


@pytest.mark.parametrize("dtype,V", [("bf16", 4096), ("f32", 2048)])
@pytest.mark.parametrize("one_hot", [False, True])
def test_emitted_tokens_follow_the_target(dtype, V, one_hot):
    z_dev, y_dev, z, y = stored_rows(dtype, V, seed=7 + V)
    p0, p1, q0 = softmax64(z[0]), softmax64(z[1]), softmax64(y)
    dev = torch.device("cuda", 0)
    target = z_dev.to(dev).unsqueeze(0).expand(PER_CALL, 2, V).contiguous()
    draft = None if one_hot else y_dev.to(dev).view(1, 1, V).expand(PER_CALL, 1, V).contiguous()
    out = (torch.empty(PER_CALL, dtype=torch.int32, device=dev),
           torch.empty(PER_CALL, 2, dtype=torch.int32, device=dev))
    rng = np.random.default_rng(1000 + V + one_hot)
    first = np.zeros(V, np.int64)
    bonus = np.zeros(V, np.int64)
    for _ in range(TRIALS // PER_CALL):
        # the drafter proposes ids from q; a one-hot drafter passes no logits,
        # so the rule sees a point mass at the id
        ids = rng.choice(V, size=PER_CALL, p=q0)
        tokens = torch.from_numpy(ids.astype(np.int32).reshape(PER_CALL, 1)).to(dev)
        uniforms = torch.from_numpy(rng.random((PER_CALL, 2), dtype=np.float32)).to(dev)
        n, t = sv.spec_verify(target, draft, tokens, None, uniforms, T, V=V, out=out)
        n, t = n.cpu().numpy(), t.cpu().numpy()
        assert np.all((n == 0) | (n == 1))
        first += np.bincount(t[:, 0], minlength=V)
        bonus += np.bincount(t[n == 1, 1], minlength=V)
    stat, bound, bins = chi2_holds(first, p0)
    assert stat < bound, f"position 0: chi2 {stat:.1f} over {bins} bins, bound {bound:.1f}"
    stat, bound, bins = chi2_holds(bonus, p1)
    assert stat < bound, f"bonus: chi2 {stat:.1f} over {bins} bins, bound {bound:.1f}"
    # the acceptance rate itself: sum_t min(p, q) with draft logits; with a
    # point mass at the proposed id, sum_t q(t) p(t)
    rate = bonus.sum() / TRIALS
    expect = float((q0 * p0).sum()) if one_hot else float(np.minimum(p0, q0).sum())
    assert abs(rate - expect) < 5.0 * np.sqrt(expect * (1 - expect) / TRIALS) + 1e-12
