"""spec_verify_accept_sim on the GPU against the oracle (acceptance
simulation: a_i, E[j], the first rejection j and the loss weights of
"今热点：让AI草稿模型学会"照镜子"", sections "VAT怎么把"验收规则"塞进训练里" and
"第二件事，改权重分配的锚点")."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import BF16, F32, make_config, make_workload
from helpers import device_inputs
from oracle import FLAG_ACCEPT_TIE, FLAG_INVALID, default as default_oracle

pytestmark = pytest.mark.gpu


def run_sim(w, decay=0.8, with_u=True):
    d = device_inputs(w)
    a, e, j, wt = sv.spec_verify_accept_sim(d["target"], d["draft"], d["tokens"], d["lens"],
                                            d["uniforms"] if with_u else None, w.temperature, decay, V=w.V)
    torch.cuda.synchronize()
    cpu = lambda t: None if t is None else t.cpu().numpy()
    return cpu(a), cpu(e), cpu(j), cpu(wt)


def oracle_sim(w, decay=0.8, with_u=True):
    orc = default_oracle()
    o = orc.verify(w.target, w.draft, w.tokens, w.lens, w.uniforms, w.temperature, False, diag=True)
    s = orc.accept_sim(o["p"], o["q"], w.tokens, w.lens, w.uniforms if with_u else None, decay, V=w.V)
    return o, s


def check(w, decay=0.8, with_u=True):
    a, e, j, wt = run_sim(w, decay, with_u)
    o, s = oracle_sim(w, decay, with_u)
    rtol = 2e-3 if w.dtype == BF16 else 1e-5
    valid = (o["flags"] & FLAG_INVALID) == 0
    L = np.where(valid, w.draft_lens, 0)
    used = (np.arange(w.k_max)[None, :] < L[:, None]) & valid[:, None]
    # a_i and E[j]
    if used.any():
        rel = np.abs(a[used] - s["a"][used]) / np.maximum(s["a"][used], 1e-30)
        assert rel.max() <= rtol, ("a", float(rel.max()))
    assert np.isnan(a[~used]).all()
    ev = valid & (L > 0)
    if ev.any():
        # a sum of up to L products of a_i: L times the per-factor bound
        rel = np.abs(e[ev] - s["e"][ev]) / np.maximum(s["e"][ev], 1e-6)
        bound = rtol * np.maximum(L[ev], 1)
        assert np.all(rel <= bound), ("E[j]", float(rel.max()))
    assert np.all(e[valid & (L == 0)] == 0.0)
    assert np.isnan(e[~valid]).all()
    if not with_u:
        assert j is None and wt is None
        return
    # first rejection: exact outside the acceptance near-tie band; inside it
    # the GPU may land on either side, and its weights must follow its own j
    tie = (o["flags"] & FLAG_ACCEPT_TIE) != 0
    assert np.array_equal(j[~valid], np.full((~valid).sum(), -1))
    sure = valid & ~tie
    assert np.array_equal(j[sure], s["j"][sure])
    assert np.array_equal(j[valid], o["len"][valid]) or tie.any()
    for b in np.flatnonzero(valid):
        jb, Lb = int(j[b]), int(L[b])
        assert 0 <= jb <= Lb
        i = np.arange(w.k_max)
        want = np.where(i >= Lb, 0.0, np.where(i <= jb, 1.0, float(decay) ** np.maximum(i - jb, 0)))
        assert np.allclose(wt[b], want, rtol=1e-6, atol=0), b
    assert np.isnan(wt[~valid]).all()


@pytest.mark.parametrize("cfg", [1, 2, 3, 5])
def test_accept_sim_configs(cfg):
    check(make_config(cfg))


def test_accept_sim_without_uniforms():
    check(make_config(2), with_u=False)


@pytest.mark.parametrize("decay", [0.0, 0.5, 1.0])
def test_accept_sim_decay(decay):
    w = make_workload(B=40, k_max=10, V=3000, dtype=F32, seed=21, boost=3.0, draft_noise=0.5)
    check(w, decay=decay)


def test_accept_sim_ragged_lengths_and_invalid():
    w = make_workload(B=9, k_max=6, V=2049, dtype=BF16, seed=22, lens=[0, 1, 6, 3, 6, 2, 4, 5, 6])
    w.lens[4] = 7                  # length > k_max: invalid
    w.lens[6] = -1                 # negative length: invalid
    w.tokens[7, 2] = 5000          # id out of range inside the length: invalid
    w.tokens[3, 4] = 99999         # beyond the length: never read
    check(w)


def test_accept_sim_matches_spec_verify_first_rejection():
    """The simulated j is the j that spec_verify returns on the same inputs."""
    w = make_config(2)
    d = device_inputs(w)
    n, _ = sv.spec_verify(d["target"], d["draft"], d["tokens"], d["lens"], d["uniforms"], w.temperature, V=w.V)
    _, _, j, _ = sv.spec_verify_accept_sim(d["target"], d["draft"], d["tokens"], d["lens"], d["uniforms"],
                                           w.temperature, 0.8, V=w.V)
    torch.cuda.synchronize()
    assert np.array_equal(n.cpu().numpy(), j.cpu().numpy())
