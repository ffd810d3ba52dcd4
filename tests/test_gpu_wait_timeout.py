"""The bound on the bulk-copy kernel's barrier waits, exercised without a GPU
fault: ``lost_copy_request`` makes the row-statistics kernel skip one stage's
copy (nothing ever completes that stage's barrier), the consumers' wait runs
out after ``wait_timeout_us``, and the request whose statistics were lost
reports -2 while the call returns normally.  The same context then runs a
clean step with the unchanged results."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import BF16, F32, make_workload
from helpers import device_inputs

pytestmark = pytest.mark.gpu
TMA = sv.StatsKernel.TMA


def verify(d, w, greedy, **kw):
    n, t = sv.spec_verify(d["target"], None if greedy else d["draft"], d["tokens"], d["lens"],
                          None if greedy else d["uniforms"], w.temperature, greedy, V=w.V,
                          stats_kernel=TMA, **kw)
    torch.cuda.synchronize()
    return n.cpu().numpy(), t.cpu().numpy()


@pytest.mark.parametrize("greedy", [False, True])
@pytest.mark.parametrize("V,dtype,victim", [(1000, F32, 2), (151936, BF16, 5)])
def test_lost_copy_times_out_and_the_context_stays_usable(V, dtype, victim, greedy):
    w = make_workload(B=12, k_max=4, V=V, dtype=dtype, seed=71, boost=4.0, draft_noise=0.3,
                      lens=[4, 3, 4, 2, 4, 4, 1, 4, 0, 4, 3, 4])
    d = device_inputs(w)
    clean = verify(d, w, greedy)
    assert np.all(clean[0] >= 0)

    # 20 ms: long against any normal wait (microseconds), short for a test
    n, t = verify(d, w, greedy, wait_timeout_us=20000, lost_copy_request=victim + 1)
    assert n[victim] == -2 and np.all(t[victim] == -1)
    # other requests: unaffected, or lost with the rest of that CTA's later work
    lost = n == -2
    assert np.all(t[lost] == -1)
    assert np.array_equal(n[~lost], clean[0][~lost]) and np.array_equal(t[~lost], clean[1][~lost])
    assert lost.sum() < w.B

    again = verify(d, w, greedy)
    assert np.array_equal(again[0], clean[0]) and np.array_equal(again[1], clean[1])


def test_lost_copy_needs_the_bulk_copy_kernel():
    w = make_workload(B=4, k_max=2, V=512, dtype=F32, seed=72)
    d = device_inputs(w)
    for kernel in (sv.StatsKernel.VEC16, sv.StatsKernel.SCALAR):
        with pytest.raises(sv.SpecVerifyError):
            sv.spec_verify(d["target"], d["draft"], d["tokens"], d["lens"], d["uniforms"], V=w.V,
                           stats_kernel=kernel, lost_copy_request=1)


def draw_victims(clean_len, w):
    """One request whose draw is a redraw after a rejection (j < L) and one
    whose draw is the bonus token (j == L)."""
    L = w.draft_lens
    resid = [b for b in range(w.B) if 0 <= clean_len[b] < L[b]]
    bonus = [b for b in range(w.B) if clean_len[b] == L[b]]
    return resid[:1] + bonus[:1]


@pytest.mark.parametrize("path", [sv.DrawPath.QUEUE, sv.DrawPath.CLUSTER])
@pytest.mark.parametrize("V,dtype,mode,misalign", [(1000, F32, "logits", False), (151936, BF16, "logits", False),
                                                   (151936, BF16, "ids", False), (4099, F32, "logits", True)])
def test_lost_draw_copy_times_out_and_the_context_stays_usable(V, dtype, mode, misalign, path):
    """The draw's waits on its own bulk copies are bounded too, on both
    draw paths: ``lost_draw_request`` makes the draw skip the first staging
    of one request's draw, that wait runs out, and the request reports -2."""
    w = make_workload(B=12, k_max=4, V=V, dtype=dtype, seed=73, boost=3.0, draft_noise=0.5, draft_mode=mode,
                      lens=[4, 3, 4, 2, 4, 4, 1, 4, 0, 4, 3, 4])
    d = device_inputs(w, misalign=misalign)
    kernel = sv.StatsKernel.SCALAR if misalign else TMA

    def run(**kw):
        n, t = sv.spec_verify(d["target"], d["draft"], d["tokens"], d["lens"], d["uniforms"], w.temperature,
                              V=w.V, stats_kernel=kernel, draw_path=path, **kw)
        torch.cuda.synchronize()
        return n.cpu().numpy(), t.cpu().numpy()

    clean = run()
    assert np.all(clean[0] >= 0)
    victims = draw_victims(clean[0], w)
    assert victims
    for victim in victims:
        n, t = run(wait_timeout_us=20000, lost_draw_request=victim + 1)
        assert n[victim] == -2 and np.all(t[victim] == -1)
        lost = n == -2
        assert np.all(t[lost] == -1)
        assert np.array_equal(n[~lost], clean[0][~lost]) and np.array_equal(t[~lost], clean[1][~lost])
        assert lost.sum() < w.B
        again = run()
        assert np.array_equal(again[0], clean[0]) and np.array_equal(again[1], clean[1])
