"""The two ways a sampling call makes its final draws give the same outputs:
the queue path (scan kernel, draw kernel over a queue of pieces, residual
selection kernel) and the cluster path (one thread-block cluster per
request: scan and draw in one kernel).  Each case runs both, forced through
``draw_path``, requires identical outputs, and compares them with the
oracle (exact, or a legal outcome where the oracle flags a near tie)."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import BF16, F32, make_config, make_workload
from helpers import compare, device_inputs, run_oracle

pytestmark = pytest.mark.gpu
PATHS = (sv.DrawPath.QUEUE, sv.DrawPath.CLUSTER)


def both_paths(w, misalign=False, stats_kernel=sv.StatsKernel.AUTO):
    d = device_inputs(w, misalign=misalign)
    outs = []
    for path in PATHS:
        n, t = sv.spec_verify(d["target"], d["draft"], d["tokens"], d["lens"], d["uniforms"], w.temperature,
                              V=w.V, stats_kernel=stats_kernel, draw_path=path)
        torch.cuda.synchronize()
        outs.append((n.cpu().numpy(), t.cpu().numpy()))
    (n0, t0), (n1, t1) = outs
    assert np.array_equal(n0, n1) and np.array_equal(t0, t1)
    o = run_oracle(w, diag=True)
    counts = compare(w, n1, t1, o, diag=o)
    assert counts["exact"] + counts["tie_ok"] == w.B
    return n1, t1


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_named_workloads_on_both_paths(cfg):
    both_paths(make_config(cfg))


@pytest.mark.parametrize("V,dtype", [(5, F32), (1000, F32), (4099, BF16), (65536, F32), (151936, BF16)])
def test_vocabularies_on_both_paths(V, dtype):
    # P = 1 (a cluster of one CTA) up to P = 19 (clusters of 8, 2-3 pieces each)
    w = make_workload(B=10, k_max=5, V=V, dtype=dtype, seed=81, boost=3.0, draft_noise=0.5,
                      lens=[5, 4, 0, 5, 3, 5, 1, 5, 2, 5])
    both_paths(w)


def test_one_hot_on_both_paths():
    w = make_workload(B=12, k_max=6, V=151936, dtype=BF16, seed=82, boost=6.0, draft_mode="ids",
                      lens_choices=(0, 3, 6), lens_probs=(0.2, 0.3, 0.5))
    both_paths(w)


def test_misaligned_rows_on_both_paths():
    w = make_workload(B=8, k_max=4, V=4099, dtype=F32, seed=83, boost=2.0, draft_noise=0.4)
    both_paths(w, misalign=True, stats_kernel=sv.StatsKernel.SCALAR)


def test_largest_vocabulary_on_both_paths():
    # P = 96 fp32 pieces: several per CTA of the cluster, more than 32 per selection warp
    w = make_workload(B=3, k_max=2, V=sv.MAX_V, dtype=F32, seed=84, z_sigma=4.0, boost=0.0, draft_noise=0.5,
                      lens=[2, 1, 2])
    both_paths(w)


def test_auto_picks_the_cluster_path_for_small_batches_only():
    small, large = make_config(4), make_config(5)
    assert sv.auto_draw_path(small.B, small.k_max, small.V, sv.BF16) == sv.DrawPath.CLUSTER
    assert sv.auto_draw_path(large.B, large.k_max, large.V, sv.F32) == sv.DrawPath.QUEUE
