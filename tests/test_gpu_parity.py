"""GPU parity on the five named workloads at their full sizes, in the launch
configuration bench.py times (default kernel choice), through the C ABI.
Every request of every workload is compared with the oracle."""
import functools

import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import make_config
from helpers import compare, compare_stats, device_inputs, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@functools.lru_cache(maxsize=None)
def workload(cfg):
    return make_config(cfg)


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_sampling_parity(cfg):
    w = workload(cfg)
    g_len, g_tok = run_gpu(w)
    o = run_oracle(w, diag=True)
    counts = compare(w, g_len, g_tok, o, diag=o)
    assert counts["exact"] + counts["tie_ok"] + counts["invalid"] == w.B
    print(f"config {cfg}: {counts}, mean accept {float(np.mean(g_len)):.3f}")


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_greedy_parity(cfg):
    w = workload(cfg)
    g_len, g_tok = run_gpu(w, greedy=True)
    o = run_oracle(w, greedy=True)
    counts = compare(w, g_len, g_tok, o, greedy=True)
    assert counts["exact"] == w.B


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_row_statistics_parity(cfg):
    w = workload(cfg)
    d = device_inputs(w)
    g = sv.spec_verify_stats(d["target"], d["draft"], d["tokens"], d["lens"], w.temperature, V=w.V)
    torch.cuda.synchronize()
    o = run_oracle(w, diag=True)
    errs = compare_stats(w, g, o)
    print(f"config {cfg}: max relative errors {errs}")


def test_repeatable_and_stream_ordered():
    w = workload(2)
    d = device_inputs(w)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = [x.clone() for x in sv.spec_verify(d["target"], d["draft"], d["tokens"], None, d["uniforms"])]
        b = [x.clone() for x in sv.spec_verify(d["target"], d["draft"], d["tokens"], None, d["uniforms"])]
    s.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_host_entry_point_matches_device_entry_point():
    w = workload(4)
    g_len, g_tok = run_gpu(w)
    tgt = torch.from_numpy(w.target)
    dft = torch.from_numpy(w.draft)
    tgt, dft = tgt.view(torch.bfloat16).pin_memory(), dft.view(torch.bfloat16).pin_memory()
    out = sv.spec_verify_host(tgt, dft, torch.from_numpy(w.tokens).pin_memory(), None,
                              torch.from_numpy(w.uniforms).pin_memory(), w.temperature)
    torch.cuda.synchronize()
    assert np.array_equal(out[0].numpy(), g_len) and np.array_equal(out[1].numpy(), g_tok)


@pytest.mark.parametrize("greedy", [False, True])
def test_host_entry_point_copies_only_the_rows_it_reads(greedy):
    """Mixed draft lengths (rows past L_b are NaN in the host tensors): the
    host entry point copies only the rows the method reads, so the staging
    rows it skips keep what they held before -- here 0xff bytes, NaN in fp32
    -- and the outputs still equal the device entry point's."""
    w = workload(5)
    g_len, g_tok = run_gpu(w, greedy=greedy)
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a)).pin_memory()
    staging = torch.full((w.target.nbytes + w.draft.nbytes + (1 << 20),), 255, dtype=torch.uint8,
                         device="cuda")
    out = sv.spec_verify_host(pin(w.target), None if greedy else pin(w.draft), pin(w.tokens), pin(w.lens),
                              None if greedy else pin(w.uniforms), w.temperature, greedy, V=w.V,
                              staging=staging)
    torch.cuda.synchronize()
    assert np.array_equal(out[0].numpy(), g_len) and np.array_equal(out[1].numpy(), g_tok)
    # the skipped rows were not written: the first padding row of a short
    # request still holds the fill bytes
    b = int(np.argmin(w.draft_lens))
    L = int(w.draft_lens[b])
    assert L < w.k_max
    row = w.target.shape[2] * w.target.itemsize
    off = (b * (w.k_max + 1) + L + 1) * row
    assert bool((staging[off:off + row] == 255).all())
