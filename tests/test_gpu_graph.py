"""A verification step captured as one CUDA graph (graph.VerifyGraph) gives
exactly the results of the direct call, and later replays follow new inputs
copied into its buffers."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.graph import VerifyGraph
from speculative_decoding_verification_92_b200.workload import make_config, make_workload
from helpers import device_inputs

pytestmark = pytest.mark.gpu


def direct(d, w, greedy=False):
    n, t = sv.spec_verify(d["target"], None if greedy else d["draft"], d["tokens"], d["lens"],
                          None if greedy else d["uniforms"], w.temperature, greedy, V=w.V)
    torch.cuda.synchronize()
    return n.cpu().numpy(), t.cpu().numpy()


@pytest.mark.parametrize("cfg,greedy", [(1, False), (1, True), (4, False), (5, False)])
def test_graph_replay_matches_direct_call(cfg, greedy):
    w = make_config(cfg)
    d = device_inputs(w)
    g = VerifyGraph(d["target"], d["draft"], d["tokens"], d["lens"], d["uniforms"], w.temperature, greedy, V=w.V)
    want = direct(d, w, greedy)
    for _ in range(3):
        n, t = g.step()
        torch.cuda.synchronize()
        assert np.array_equal(n.cpu().numpy(), want[0]) and np.array_equal(t.cpu().numpy(), want[1])


def test_graph_replay_follows_new_inputs():
    shape = dict(B=16, k_max=6, V=4096, dtype="bf16", boost=3.0, draft_noise=0.4,
                 lens_choices=(0, 3, 6), lens_probs=(0.2, 0.3, 0.5))
    w0 = make_workload(seed=31, **shape)
    d0 = device_inputs(w0)
    g = VerifyGraph(d0["target"], d0["draft"], d0["tokens"], d0["lens"], d0["uniforms"], w0.temperature, V=w0.V)
    for seed in (32, 33, 34):
        w = make_workload(seed=seed, **shape)
        d = device_inputs(w)
        n, t = g.step(**d)
        torch.cuda.synchronize()
        want = direct(d, w)
        assert np.array_equal(n.cpu().numpy(), want[0]) and np.array_equal(t.cpu().numpy(), want[1])
