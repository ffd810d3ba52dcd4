"""spec_verify_static_scratch: the allocation-free entry point.

Some callers cannot give the library device memory of its own (a stream being
captured into a CUDA graph, hosts without a device allocator, services that
forbid allocations after start-up).  For them the library keeps its scratch in
a fixed array inside the library.  These tests call that entry point through
the C ABI (ctypes, raw device pointers, no workspace argument) and check that
it returns exactly what spec_verify with a caller-provided workspace returns,
on two calls in a row with different problems (the shared array keeps the
previous call's contents, which must not leak into the next call).  This file
is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200 import Status, _Shape
from speculative_decoding_verification_92_b200.workload import make_config, make_workload
from helpers import device_inputs, run_gpu

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 1 << 20


def call_static(w, d, greedy=False):
    """spec_verify_static_scratch through the C ABI; returns (status, len, tokens)."""
    lib = sv.library()
    dt = sv.BF16 if w.dtype == "bf16" else sv.F32
    shape = _Shape(w.B, w.k_max, w.V, dt, w.row_stride)
    out_len = torch.full((w.B,), -7, dtype=torch.int32, device="cuda")
    out_tok = torch.full((w.B, w.k_max + 1), -7, dtype=torch.int32, device="cuda")
    ptr = lambda t: None if t is None else t.data_ptr()
    st = lib.spec_verify_static_scratch(
        ctypes.byref(shape), ptr(d["target"]), None if greedy else ptr(d["draft"]), ptr(d["tokens"]),
        ptr(d["lens"]), None if greedy else ptr(d["uniforms"]), w.temperature, int(greedy),
        ptr(out_len), ptr(out_tok), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return st, out_len.cpu().numpy(), out_tok.cpu().numpy()


def test_static_scratch_matches_workspace_entry_point_on_consecutive_calls():
    w1 = make_config(2)                                   # 64 x 17 rows x 19 pieces of partials
    w2 = make_workload(B=33, k_max=12, V=20000, dtype="f32", seed=5, boost=4.0, draft_noise=0.3,
                       lens_choices=(0, 4, 12), lens_probs=(0.4, 0.3, 0.3))
    w3 = make_config(4)                                   # a small batch: the cluster draw path
    assert sv.workspace_bytes(w1.B, w1.k_max, w1.V, sv.BF16) <= SCRATCH_BYTES
    for w in (w1, w2, w3, w1):
        d = device_inputs(w)
        want_len, want_tok = run_gpu(w, inputs=d)
        st, got_len, got_tok = call_static(w, d)
        assert st == Status.OK
        assert np.array_equal(got_len, want_len) and np.array_equal(got_tok, want_tok)
        g_len, g_tok = run_gpu(w, greedy=True, inputs=d)
        st, got_len, got_tok = call_static(w, d, greedy=True)
        assert st == Status.OK
        assert np.array_equal(got_len, g_len) and np.array_equal(got_tok, g_tok)


def test_static_scratch_rejects_problems_larger_than_its_array():
    w = make_workload(B=600, k_max=16, V=64, dtype="f32", seed=6)   # fits: 600 * 33 rows * 1 piece * 8 B + draw queue
    assert sv.workspace_bytes(w.B, w.k_max, w.V, sv.F32) <= SCRATCH_BYTES
    lib = sv.library()
    big = _Shape(4096, 64, 151936, sv.BF16, 0)                      # partials far beyond 1 MiB
    assert sv.workspace_bytes(4096, 64, 151936, sv.BF16) > SCRATCH_BYTES
    st = lib.spec_verify_static_scratch(ctypes.byref(big), 0x10000, 0x10000, 0x10000, None, 0x10000, 1.0, 0,
                                        0x10000, 0x10000, None)
    assert st == Status.ESCRATCH
    assert lib.spec_verify_status_string(int(Status.ESCRATCH)).startswith(b"problem larger")
    # a shape that fits still works after the rejection
    d = device_inputs(w)
    st, got_len, got_tok = call_static(w, d)
    want_len, want_tok = run_gpu(w, inputs=d)
    assert st == Status.OK and np.array_equal(got_len, want_len) and np.array_equal(got_tok, want_tok)
