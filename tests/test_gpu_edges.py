"""GPU edge cases against the oracle: every row-statistics kernel, ragged
vocabulary tails, tiny and single-token vocabularies, empty drafts, padded
and misaligned rows, temperatures, greedy ties across piece boundaries,
extreme uniforms, invalid ids / lengths, large batches split over several
launches, the largest vocabulary and draft length, and closed forms of the
rule."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import BF16, F32, f32_to_bf16_bits, make_workload
from helpers import compare, compare_stats, device_inputs, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

KERNELS = [sv.StatsKernel.TMA, sv.StatsKernel.VEC16, sv.StatsKernel.SCALAR]


def check(w, greedy=False, kernels=KERNELS, misalign=False):
    o = run_oracle(w, greedy=greedy, diag=not greedy)
    for k in kernels:
        g_len, g_tok = run_gpu(w, greedy=greedy, stats_kernel=k, misalign=misalign)
        compare(w, g_len, g_tok, o, greedy=greedy, diag=None if greedy else o)
    return o


@pytest.mark.parametrize("dtype", [F32, BF16])
@pytest.mark.parametrize("V", [1, 5, 8, 1000, 1001, 1003, 4099, 65536, 151936])
def test_vocabulary_sizes(dtype, V):
    stride = V if (V * (4 if dtype == F32 else 2)) % 16 == 0 else V + (8 - V % 8)
    w = make_workload(B=6, k_max=3, V=V, dtype=dtype, seed=V, z_sigma=1.5, boost=3.0,
                      draft_noise=0.5, row_stride=stride)
    check(w)
    check(w, greedy=True)


@pytest.mark.parametrize("dtype", [F32, BF16])
def test_misaligned_rows_use_element_loads(dtype):
    w = make_workload(B=5, k_max=4, V=3000, dtype=dtype, seed=3, z_sigma=1.0, boost=4.0, draft_noise=0.4)
    check(w, kernels=[sv.StatsKernel.AUTO, sv.StatsKernel.SCALAR], misalign=True)
    d = device_inputs(w, misalign=True)
    with pytest.raises(sv.SpecVerifyError):
        sv.spec_verify(d["target"], d["draft"], d["tokens"], None, d["uniforms"],
                       stats_kernel=sv.StatsKernel.TMA)


def test_padded_row_stride_with_nan_columns():
    w = make_workload(B=7, k_max=5, V=2000, dtype=BF16, seed=4, boost=5.0, row_stride=2056)
    assert (w.target[0, 0, 2000:] == 0x7FC0).all()   # bf16 NaN padding columns
    check(w)


@pytest.mark.parametrize("T", [0.25, 0.6, 1.0, 2.0])
def test_temperatures(T):
    w = make_workload(B=8, k_max=6, V=5000, dtype=F32, temperature=T, seed=5, z_sigma=1.5,
                      boost=6.0, draft_noise=0.2)
    check(w, kernels=[sv.StatsKernel.AUTO])


def test_empty_drafts_and_k_zero():
    w = make_workload(B=9, k_max=4, V=777, dtype=F32, seed=6, lens=[0] * 9, row_stride=780)
    o = check(w)
    assert np.all(o["len"] == 0)
    w0 = make_workload(B=5, k_max=0, V=999, dtype=BF16, seed=7, draft_mode="ids", row_stride=1000)
    check(w0)
    check(w0, greedy=True)
    w1 = make_workload(B=5, k_max=1, V=3001, dtype=BF16, seed=8, row_stride=3008)
    check(w1)


def test_mixed_lengths_with_nan_padding_rows():
    w = make_workload(B=64, k_max=12, V=4096, dtype=F32, seed=9, boost=5.0,
                      lens_choices=(0, 4, 12), lens_probs=(0.5, 0.3, 0.2))
    assert np.isnan(w.target[w.lens == 0][:, 1]).all()
    check(w)
    check(w, greedy=True)


def test_one_hot_drafts_long_k():
    w = make_workload(B=16, k_max=64, V=2048, dtype=BF16, seed=10, boost=6.0, draft_mode="ids",
                      fav_prob=0.95)
    check(w)


def test_identical_draft_accepts_everything():
    w = make_workload(B=8, k_max=7, V=10000, dtype=F32, seed=11)
    w.draft[:] = w.target[:, :7]
    w.uniforms[:, :7] = np.float32(np.nextafter(np.float32(1), np.float32(0)))
    g_len, _ = run_gpu(w)
    assert np.all(g_len == 7)


def test_zero_probability_draft_rejects():
    w = make_workload(B=4, k_max=3, V=300, dtype=F32, seed=12, draft_mode="ids")
    for b in range(4):
        w.target[b, 0, w.tokens[b, 0]] = -np.inf
    w.uniforms[:, 0] = 0.0
    g_len, g_tok = run_gpu(w)
    assert np.all(g_len == 0)
    assert np.all(g_tok[:, 0] != w.tokens[:, 0])
    o = run_oracle(w, diag=True)
    compare(w, g_len, g_tok, o, diag=o)


@pytest.mark.parametrize("u", [0.0, 1e-7, 0.5, float(np.nextafter(np.float32(1), np.float32(0)))])
def test_extreme_uniforms(u):
    w = make_workload(B=12, k_max=4, V=1500, dtype=F32, seed=13, boost=2.0, draft_noise=0.6)
    w.uniforms[:] = np.float32(u)
    o = run_oracle(w, diag=True)
    g_len, g_tok = run_gpu(w)
    compare(w, g_len, g_tok, o, diag=o)


def test_greedy_ties_across_piece_boundaries():
    V = 151936
    w = make_workload(B=3, k_max=2, V=V, dtype=BF16, seed=14, draft_mode="ids")
    CE = 3 * 8192  # three bf16 pieces of 16 KiB: CE - 1 and CE sit in pieces 2 and 3
    for b in range(3):
        for i in range(3):
            row = np.zeros(V, np.float32)
            row[[CE - 1, CE, 5 * CE + 3, V - 1]] = 9.0   # four-way tie
            w.target[b, i] = f32_to_bf16_bits(row)
    w.tokens[0] = [CE - 1, CE - 1]
    w.tokens[1] = [CE, CE - 1]
    w.tokens[2] = [CE - 1, V - 1]
    g_len, g_tok = run_gpu(w, greedy=True)
    assert list(g_len) == [2, 0, 1]
    assert list(g_tok[0]) == [CE - 1, CE - 1, CE - 1]
    assert list(g_tok[1]) == [CE - 1, -1, -1]
    assert list(g_tok[2]) == [CE - 1, CE - 1, -1]
    check(w, greedy=True)


def test_invalid_requests_are_reported_not_read():
    w = make_workload(B=6, k_max=3, V=500, dtype=F32, seed=15, lens=[3, 3, 2, 3, 3, 1])
    w.tokens[0, 1] = 500          # id == V
    w.tokens[1, 0] = -3           # negative id
    w.tokens[2, 2] = 10**6        # beyond the request's length: never read
    w.lens[3] = 4                 # length > k_max
    w.lens[4] = -1
    o = run_oracle(w, diag=True)
    assert list(o["len"][[0, 1, 3, 4]]) == [-1, -1, -1, -1]
    g_len, g_tok = run_gpu(w)
    compare(w, g_len, g_tok, o, diag=o)
    assert list(g_len[[0, 1, 3, 4]]) == [-1, -1, -1, -1]
    assert g_len[2] >= 0 and g_len[5] >= 0


@pytest.mark.parametrize("dtype", [F32, BF16])
def test_largest_vocabulary(dtype):
    # V = MAX_V: 96 pieces of 16 KiB per fp32 row (48 per bf16 row), so the
    # selection sums more than 32 pieces per draw
    # heavy-tailed logits (sigma 4): the mass sits on a few hundred ids spread
    # over the whole row, so most draws are far from a near-tie and compare
    # exactly, while the piece and segment sums still span every piece
    w = make_workload(B=6, k_max=2, V=sv.MAX_V, dtype=dtype, seed=61, z_sigma=4.0, boost=0.0,
                      draft_noise=0.5, lens=[2, 1, 0, 2, 2, 1])
    o = check(w)
    assert np.count_nonzero(o["flags"] & 3) <= 2
    check(w, greedy=True)


def test_largest_draft_length():
    # k_max = MAX_K: four drafts per draw-kernel thread; one request accepts
    # all 1024 drafts (identical draft, bonus from row 1024), the others stop
    # early or at their own length
    w = make_workload(B=3, k_max=sv.MAX_K, V=256, dtype=F32, seed=62, boost=3.0, draft_noise=0.3,
                      lens=[sv.MAX_K, 1000, 517])
    w.draft[0] = w.target[0, :sv.MAX_K]
    check(w)
    check(w, greedy=True)
    g_len, _ = run_gpu(w)
    assert g_len[0] == sv.MAX_K


def test_many_requests_span_several_launches():
    w = make_workload(B=5000, k_max=2, V=96, dtype=BF16, seed=16, boost=2.0, draft_noise=0.5,
                      lens_choices=(0, 1, 2), lens_probs=(0.3, 0.3, 0.4))
    check(w, kernels=[sv.StatsKernel.TMA, sv.StatsKernel.VEC16])


def test_stats_on_ragged_and_unaligned_rows():
    w = make_workload(B=4, k_max=3, V=1003, dtype=F32, seed=17, boost=2.0, row_stride=1004)
    d = device_inputs(w)
    o = run_oracle(w, diag=True)
    for k in KERNELS:
        g = sv.spec_verify_stats(d["target"], d["draft"], d["tokens"], None, w.temperature, V=w.V,
                                 stats_kernel=k)
        torch.cuda.synchronize()
        compare_stats(w, g, o)
