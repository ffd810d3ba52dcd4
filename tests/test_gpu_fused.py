"""The one-launch path (StatsKernel.FUSED): statistics, scan and draw in one
persistent kernel.  Same comparison rule as the two-kernel path: exact
outcomes against the oracle except flagged near-ties, which must be legal."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import BF16, F32, make_config, make_workload
from helpers import compare, device_inputs, run_gpu, run_oracle

pytestmark = pytest.mark.gpu
FUSED = sv.StatsKernel.FUSED


def check(w, **kw):
    g_len, g_tok = run_gpu(w, stats_kernel=FUSED, **kw)
    o = run_oracle(w, diag=True)
    compare(w, g_len, g_tok, o, diag=o)
    return g_len, g_tok


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_fused_configs(cfg):
    check(make_config(cfg))


def test_fused_is_deterministic_and_matches_the_two_kernel_path_outside_ties():
    w = make_config(2)
    d = device_inputs(w)
    runs = [run_gpu(w, stats_kernel=FUSED, inputs=d) for _ in range(3)]
    for n, t in runs[1:]:
        assert np.array_equal(n, runs[0][0]) and np.array_equal(t, runs[0][1])
    n2, t2 = run_gpu(w, stats_kernel=sv.StatsKernel.TMA, inputs=d)
    o = run_oracle(w)
    sure = (o["flags"] & 3) == 0
    assert np.array_equal(runs[0][0][sure], n2[sure]) and np.array_equal(runs[0][1][sure], t2[sure])


@pytest.mark.parametrize("V,dtype", [(1, F32), (5, BF16), (1000, F32), (4099, BF16), (65536, BF16), (20000, F32)])
def test_fused_vocab_sizes(V, dtype):
    es = 4 if dtype == F32 else 2
    stride = V if (V * es) % 16 == 0 else V + (16 // es - V % (16 // es))
    w = make_workload(B=24, k_max=5, V=V, dtype=dtype, seed=41 + V, boost=2.0, draft_noise=0.5,
                      row_stride=stride, lens_choices=(0, 2, 5), lens_probs=(0.2, 0.3, 0.5))
    check(w)


def test_fused_one_hot_and_extreme_uniforms():
    w = make_workload(B=32, k_max=8, V=3000, dtype=BF16, seed=44, draft_mode="ids", fav_prob=0.7, boost=4.0)
    check(w)
    w.uniforms[:] = np.float32(0.0)
    check(w)
    w.uniforms[:] = np.float32(np.nextafter(np.float32(1), np.float32(0)))
    check(w)


def test_fused_identical_draft_accepts_everything():
    w = make_workload(B=16, k_max=6, V=2048, dtype=F32, seed=45, draft_noise=0.0)
    g_len, _ = check(w)
    assert np.all(g_len == w.draft_lens)


def test_fused_invalid_requests():
    w = make_workload(B=8, k_max=4, V=700, dtype=F32, seed=46, lens=[4, 4, 3, 4, 2, 4, 0, 1])
    w.tokens[0, 1] = 700
    w.tokens[1, 0] = -5
    w.lens[3] = 5
    w.lens[5] = -1
    w.tokens[2, 3] = 10 ** 6      # beyond the length: never read
    g_len, g_tok = check(w)
    assert list(g_len[[0, 1, 3, 5]]) == [-1, -1, -1, -1]
    assert np.all(g_tok[[0, 1, 3, 5]] == -1)


def test_fused_many_requests():
    w = make_workload(B=1500, k_max=3, V=512, dtype=BF16, seed=47, boost=1.0, draft_noise=0.3,
                      lens_choices=(0, 1, 3), lens_probs=(0.3, 0.3, 0.4))
    check(w)


def test_fused_rejects_what_it_cannot_run():
    w = make_config(1)
    with pytest.raises(sv.SpecVerifyError):      # unaligned rows
        run_gpu(w, stats_kernel=FUSED, misalign=True)
    with pytest.raises(sv.SpecVerifyError):      # greedy
        run_gpu(w, greedy=True, stats_kernel=FUSED)
