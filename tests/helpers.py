"""Shared helpers of the GPU parity tests: move a seeded workload to the
device, run the library and the oracle on the same inputs, and compare.

Comparison rule: accept lengths and emitted ids must match exactly, except
for requests the oracle flags as near-ties (|u_i - a_i| < 1e-5 at an examined
position, or u*W within 1e-5 W of a CDF step of the final draw).  For those
the GPU's outcome must still be a legal one: its accepted prefix equals the
drafts, any disagreement about j sits at a flagged position, the emitted
token has positive weight, and a different draw lies next to the oracle's on
the CDF (only weight of at most 2e-5 W between them).
"""
from __future__ import annotations

import numpy as np
import torch

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200.workload import BF16, bf16_bits_to_f32
from oracle import FLAG_ACCEPT_TIE, FLAG_DRAW_TIE, FLAG_INVALID
from oracle import default as default_oracle

TIE = 1e-5


def to_torch(a: np.ndarray, dtype: str | None = None, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == BF16:
        t = t.view(torch.bfloat16)
    return t.to(device)


def device_inputs(w, device="cuda", misalign=False):
    """Device tensors of a workload; misalign=True shifts the logit buffers
    by one element so that no row starts on a 16-byte boundary."""
    def logits(a):
        if a is None:
            return None
        t = to_torch(a, w.dtype, device)
        if misalign:
            flat = torch.empty(t.numel() + 1, dtype=t.dtype, device=device)
            view = flat[1:].view(t.shape)
            view.copy_(t)
            return view
        return t
    return dict(
        target=logits(w.target), draft=logits(w.draft),
        tokens=to_torch(w.tokens, device=device),
        lens=None if w.lens is None else to_torch(w.lens, device=device),
        uniforms=to_torch(w.uniforms, device=device))


def run_gpu(w, greedy=False, stats_kernel=sv.StatsKernel.AUTO, misalign=False, inputs=None, **kw):
    d = inputs if inputs is not None else device_inputs(w, misalign=misalign)
    n, t = sv.spec_verify(d["target"], None if greedy else d["draft"], d["tokens"], d["lens"],
                          None if greedy else d["uniforms"], w.temperature, greedy, V=w.V,
                          stats_kernel=stats_kernel, **kw)
    torch.cuda.synchronize()
    return n.cpu().numpy(), t.cpu().numpy()


def run_oracle(w, greedy=False, diag=False):
    return default_oracle().verify(w.target, None if greedy else w.draft, w.tokens, w.lens,
                                   None if greedy else w.uniforms.astype(np.float64),
                                   w.temperature, greedy, V=w.V, diag=diag)


def _row_f64(w, which, b, i):
    a = w.target if which == "t" else w.draft
    row = a[b, i, :w.V]
    row = bf16_bits_to_f32(row) if w.dtype == BF16 else row
    return row.astype(np.float64)


def _softmax(z):
    z = z - np.max(z)
    e = np.exp(z)
    return e / e.sum()


def draw_weights(w, b, j):
    """Weights of the final draw on row j (test-side, float64) for the
    validity check of flagged requests."""
    L = int(w.draft_lens[b])
    p = _softmax(_row_f64(w, "t", b, j) / w.temperature)
    if j == L:
        return p
    if w.draft is not None:
        q = _softmax(_row_f64(w, "d", b, j) / w.temperature)
        r = np.maximum(p - q, 0.0)
    else:
        r = p.copy()
        r[w.tokens[b, j]] = max(0.0, r[w.tokens[b, j]] - 1.0)
    return r if r.sum() > 0 else p


def compare(w, g_len, g_tok, o, greedy=False, diag=None):
    """Assert parity of every request; returns counts by outcome."""
    counts = {"exact": 0, "invalid": 0, "tie_ok": 0}
    for b in range(w.B):
        gj, oj = int(g_len[b]), int(o["len"][b])
        flags = int(o["flags"][b])
        if flags & FLAG_INVALID:
            assert gj == -1 and np.all(g_tok[b] == -1), (b, gj, g_tok[b])
            counts["invalid"] += 1
            continue
        if gj == oj and np.array_equal(g_tok[b], o["tokens"][b]):
            counts["exact"] += 1
            continue
        assert not greedy, f"greedy request {b}: gpu {gj} {g_tok[b]} vs oracle {oj} {o['tokens'][b]}"
        assert flags & (FLAG_ACCEPT_TIE | FLAG_DRAW_TIE), (
            f"request {b}: gpu (j={gj}, tok={g_tok[b][gj] if gj >= 0 else None}) vs oracle "
            f"(j={oj}, tok={o['tokens'][b][oj]}) and the oracle saw no near tie")
        L = int(w.draft_lens[b])
        assert 0 <= gj <= L
        assert np.array_equal(g_tok[b, :gj], w.tokens[b, :gj])
        assert np.all(g_tok[b, gj + 1:] == -1)
        if gj != oj:
            assert flags & FLAG_ACCEPT_TIE and diag is not None
            i = min(gj, oj)
            a = min(1.0, diag["p"][b, i] / diag["q"][b, i])
            assert abs(float(w.uniforms[b, i]) - a) < TIE, (b, i, w.uniforms[b, i], a)
        wts = draw_weights(w, b, gj)
        t = int(g_tok[b, gj])
        assert 0 <= t < w.V and wts[t] > 0, (b, gj, t)
        if gj == oj:
            assert flags & FLAG_DRAW_TIE
            to = int(o["tokens"][b, oj])
            lo, hi = min(t, to), max(t, to)
            W = wts.sum()
            assert wts[lo + 1:hi].sum() <= 2 * TIE * W, (b, t, to)
            cdf_at = wts[:hi].sum()
            assert abs(float(w.uniforms[b, w.k_max]) * W - cdf_at) <= 2 * TIE * W
        counts["tie_ok"] += 1
    return counts


def compare_stats(w, g, o, rtol=None):
    """Per-row lse / p / q against the oracle's diagnostics; returns the
    largest relative errors seen."""
    lse_t, lse_d, p, q = (x.cpu().numpy().astype(np.float64) for x in g)
    if rtol is None:
        rtol = 2e-3 if w.dtype == BF16 else 1e-5
    errs = {}
    valid = (o["flags"] & FLAG_INVALID) == 0
    L = w.draft_lens
    K = w.k_max
    used_t = (np.arange(K + 1)[None, :] <= L[:, None]) & valid[:, None]
    used_d = (np.arange(K)[None, :] < L[:, None]) & valid[:, None]
    for name, gv, ov, used in (("lse_t", lse_t, o["lse_t"], used_t), ("p", p, o["p"], used_d),
                               ("q", q, o["q"], used_d)):
        if used.any():
            rel = np.abs(gv[used] - ov[used]) / np.maximum(np.abs(ov[used]), 1e-30)
            errs[name] = float(rel.max())
            assert rel.max() <= rtol, (name, float(rel.max()), rtol)
        assert np.all(np.isnan(gv[~used])), f"{name}: unused entries must be NaN"
    if w.draft is not None and used_d.any():
        rel = np.abs(lse_d[used_d] - o["lse_d"][used_d]) / np.abs(o["lse_d"][used_d])
        errs["lse_d"] = float(rel.max())
        assert rel.max() <= rtol
        assert np.all(np.isnan(lse_d[~used_d]))
    return errs
