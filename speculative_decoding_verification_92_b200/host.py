"""ctypes binding of the host-side components in ``include/sv_host.h``.

Every class wraps one C handle of ``libspecverify.so`` (argument marshalling
only; the logic lives in ``csrc/sv_host.cpp``).  Token sequences are passed
as int32 numpy arrays (anything ``numpy.asarray`` accepts)."""
from __future__ import annotations

import ctypes

import numpy as np

from . import library

_I32, _I64, _F64, _VP = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p

_HOST_SIGNATURES = {
    "sv_ngram_create": (_VP, [_I32, _I32]),
    "sv_ngram_destroy": (None, [_VP]),
    "sv_ngram_begin_step": (None, [_VP]),
    "sv_ngram_add": (_I32, [_VP, _I64, _VP, _I64]),
    "sv_ngram_draft": (_I32, [_VP, _I64, _VP, _I64, _I32, _VP]),
    "sv_ngram_candidates": (_I32, [_VP, _I64, _VP, _I64, _I32, _VP]),
    "sv_ngram_rollouts": (_I64, [_VP]),
    "sv_ngram_tokens": (_I64, [_VP]),
    "sv_suffix_create": (_VP, [_I32]),
    "sv_suffix_destroy": (None, [_VP]),
    "sv_suffix_clear": (None, [_VP]),
    "sv_suffix_append": (_I32, [_VP, _I64, _I64, _VP, _I64]),
    "sv_suffix_draft": (_I32, [_VP, _I64, _VP, _I64, _I32, _VP]),
    "sv_suffix_candidates": (_I32, [_VP, _I64, _VP, _I64, _I32, _VP]),
    "sv_ngram_draft_batch": (_I32, [_VP, _I32, _VP, _VP, _VP, _I32, _VP, _I32, _VP, _VP]),
    "sv_suffix_draft_batch": (_I32, [_VP, _I32, _VP, _VP, _VP, _I32, _VP, _I32, _VP, _VP]),
    "sv_prefetch_create": (_VP, [_I32, _I32, _I32]),
    "sv_prefetch_destroy": (None, [_VP]),
    "sv_prefetch_observe": (_I32, [_VP, _I32, _I32]),
    "sv_prefetch_estimates": (_I32, [_VP, _VP, _VP]),
    "sv_prefetch_allocate": (_F64, [_VP, _I32, _VP]),
    "sv_roofline_work": (_I32, [_VP, _F64, _F64, _F64, _VP, _VP]),
    "sv_roofline_time": (_F64, [_VP, _VP, _F64, _F64, _F64]),
    "sv_roofline_fit": (_I32, [_VP, _I32, _VP, _VP, _VP, _VP, _VP, _VP]),
    "sv_spec_speedup": (_F64, [_VP, _VP, _VP, _VP, _F64, _I32, _F64, _F64]),
    "sv_ngram_prefetch": (_I32, [_VP, _I64, _VP, _I64, _VP, _I32, _VP, _I32, _I32, _VP, _VP, _VP, _VP]),
    "sv_prefetch_find": (_I32, [_VP, _VP, _I32, _I32, _I32]),
    "sv_draft_len_create": (_VP, [_VP, _I32, _F64, _F64, _I32]),
    "sv_draft_len_destroy": (None, [_VP]),
    "sv_draft_len_current": (_I32, [_VP]),
    "sv_draft_len_update": (_I32, [_VP, _F64]),
    "sv_block_efficiency": (_F64, [_VP, _I64]),
    "sv_spec_switch": (_I32, [_VP, _F64, _F64]),
    "sv_length_classes": (_I32, [_VP, _I64, _VP, _VP, _VP]),
    "sv_interleave_ranks": (_I32, [_VP, _I64, _I32, _VP]),
}

_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = library()
        for name, (res, args) in _HOST_SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _tok(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32).reshape(-1))


def _tail(a, n: int) -> np.ndarray:
    """The last n tokens of a context (a lookup never reads further back);
    sliced before conversion when the context supports it."""
    try:
        if len(a) > n:
            a = a[-n:]
    except TypeError:
        pass
    return _tok(a)[-n:]


def _draft_batch_flat(fn, h, ids, flat, offsets, k_max, max_lens, n_threads):
    """Batched drafting on contexts already laid out in one int32 buffer:
    request b's context is flat[offsets[b]:offsets[b+1]].  No per-request
    Python work, so the C++ lookups set the pace."""
    ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int64).reshape(-1))
    B = ids.size
    flat = np.ascontiguousarray(np.asarray(flat, dtype=np.int32).reshape(-1))
    off = np.ascontiguousarray(np.asarray(offsets, dtype=np.int64).reshape(-1))
    if off.size != B + 1:
        raise ValueError(f"{B} ids need {B + 1} offsets, got {off.size}")
    if B and (off[0] < 0 or np.any(np.diff(off) < 0) or off[-1] > flat.size):
        raise ValueError("offsets must be non-decreasing and inside the buffer")
    caps = None
    if max_lens is not None:
        caps = np.ascontiguousarray(np.asarray(max_lens, dtype=np.int32).reshape(-1))
        if caps.size != B:
            raise ValueError(f"{B} ids but {caps.size} max_lens")
    tokens = np.empty((B, int(k_max)), np.int32)
    lens = np.empty(B, np.int32)
    rc = fn(h, B, ids.ctypes.data, flat.ctypes.data if flat.size else None, off.ctypes.data, int(k_max),
            None if caps is None else caps.ctypes.data, int(n_threads),
            tokens.ctypes.data if tokens.size else None, lens.ctypes.data)
    if rc != 0:
        raise ValueError("batched drafting rejected its arguments")
    return tokens, lens


def _draft_batch(fn, h, ids, contexts, k_max, max_lens, n_threads, tail):
    """Shared marshalling of the batched drafting calls: returns the
    drafted-id array [B, k_max] (-1 padded) and the lengths [B], both int32,
    in the layout spec_verify takes as draft_tokens / draft_lens.  Only the
    last ``tail`` tokens of each context can take part in a match, so only
    those are passed."""
    ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int64).reshape(-1))
    B = ids.size
    if len(contexts) != B:
        raise ValueError(f"{B} ids but {len(contexts)} contexts")
    contexts = [c[-tail:] if len(c) > tail else c for c in contexts]
    off = np.zeros(B + 1, np.int64)
    np.cumsum(np.fromiter((len(c) for c in contexts), np.int64, count=B), out=off[1:])
    # one concatenation (and one conversion to int32) for the whole batch
    parts = [c for c in contexts if len(c)]          # an empty list would come in as float64
    flat = np.concatenate(parts, dtype=np.int32, casting="same_kind") if parts else np.zeros(1, np.int32)
    if flat.size != off[-1]:
        raise ValueError("every context must be a flat sequence of token ids")
    caps = None
    if max_lens is not None:
        caps = np.ascontiguousarray(np.asarray(max_lens, dtype=np.int32).reshape(-1))
        if caps.size != B:
            raise ValueError(f"{B} ids but {caps.size} max_lens")
    tokens = np.empty((B, int(k_max)), np.int32)
    lens = np.empty(B, np.int32)
    rc = fn(h, B, ids.ctypes.data, flat.ctypes.data, off.ctypes.data, int(k_max),
            None if caps is None else caps.ctypes.data, int(n_threads),
            tokens.ctypes.data if tokens.size else None, lens.ctypes.data)
    if rc != 0:
        raise ValueError("batched drafting rejected its arguments")
    return tokens, lens


class _Handle:
    _destroy = ""

    def __init__(self, h):
        if not h:
            raise ValueError(f"{type(self).__name__}: invalid arguments")
        self._h = h

    def close(self):
        if getattr(self, "_h", None):
            getattr(_L(), self._destroy)(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class NgramDrafter(_Handle):
    """Per-prompt n-gram drafter over the rollouts of the last ``window``
    training steps (longest match up to ``max_n``, most recent occurrence)."""
    _destroy = "sv_ngram_destroy"

    def __init__(self, max_n: int = 6, window: int = 4):
        super().__init__(_L().sv_ngram_create(int(max_n), int(window)))
        self.max_n = int(max_n)     # the longest context tail a lookup can use

    def begin_step(self):
        _L().sv_ngram_begin_step(self._h)

    def add(self, prompt_id: int, tokens):
        t = _tok(tokens)
        if _L().sv_ngram_add(self._h, int(prompt_id), t.ctypes.data, t.size) != 0:
            raise ValueError("sv_ngram_add rejected its arguments")

    def draft(self, prompt_id: int, context, k: int = 16) -> np.ndarray:
        c = _tail(context, self.max_n)
        out = np.empty(max(int(k), 1), np.int32)
        n = _L().sv_ngram_draft(self._h, int(prompt_id), c.ctypes.data, c.size, int(k), out.ctypes.data)
        if n < 0:
            raise ValueError("sv_ngram_draft rejected its arguments")
        return out[:n].copy()

    def prefetch(self, prompt_id: int, context, draft, f, k: int = 16, max_entries=None) -> dict:
        """Next drafts for the verification outcomes that the allocation
        ``f`` (one entry per branch j = 0..len(draft)) covers, drafted before
        the outcome is known: ``{(j, b): ids}`` (sv_ngram_prefetch)."""
        c, d = _tail(context, self.max_n), _tok(draft)
        fa = np.ascontiguousarray(np.asarray(f, dtype=np.int32).reshape(-1))
        if fa.size != d.size + 1:
            raise ValueError(f"f needs {d.size + 1} entries (branches j = 0..{d.size}), got {fa.size}")
        cap = int(fa.clip(min=0).sum()) if max_entries is None else int(max_entries)
        oj, ob, ol = (np.empty(max(cap, 1), np.int32) for _ in range(3))
        ot = np.empty((max(cap, 1), max(int(k), 1)), np.int32)
        n = _L().sv_ngram_prefetch(self._h, int(prompt_id), c.ctypes.data, c.size, d.ctypes.data, d.size,
                                   fa.ctypes.data, int(k), cap, oj.ctypes.data, ob.ctypes.data, ot.ctypes.data,
                                   ol.ctypes.data)
        if n < 0:
            raise ValueError("sv_ngram_prefetch rejected its arguments")
        return {(int(oj[e]), int(ob[e])): ot[e, :ol[e]].copy() for e in range(n)}

    def draft_batch(self, prompt_ids, contexts, k_max: int, max_lens=None, n_threads: int = 0):
        """Drafts for a whole batch in one call: ``(draft_tokens [B, k_max],
        draft_lens [B])`` int32, -1 padded, ready for spec_verify without
        draft logits.  ``max_lens`` caps each request (controller length or
        budget); ``n_threads`` 0 uses the hardware threads."""
        return _draft_batch(_L().sv_ngram_draft_batch, self._h, prompt_ids, contexts, k_max, max_lens, n_threads,
                            self.max_n)

    def draft_batch_flat(self, prompt_ids, flat, offsets, k_max: int, max_lens=None, n_threads: int = 0):
        """draft_batch on contexts laid out back to back in one int32 buffer
        (request b: flat[offsets[b]:offsets[b+1]])."""
        return _draft_batch_flat(_L().sv_ngram_draft_batch, self._h, prompt_ids, flat, offsets, k_max, max_lens,
                                 n_threads)

    def candidates(self, prompt_id: int, context, f: int) -> np.ndarray:
        c = _tail(context, self.max_n)
        out = np.empty(max(int(f), 1), np.int32)
        n = _L().sv_ngram_candidates(self._h, int(prompt_id), c.ctypes.data, c.size, int(f), out.ctypes.data)
        if n < 0:
            raise ValueError("sv_ngram_candidates rejected its arguments")
        return out[:n].copy()

    @property
    def rollouts(self) -> int:
        return int(_L().sv_ngram_rollouts(self._h))

    @property
    def tokens(self) -> int:
        return int(_L().sv_ngram_tokens(self._h))


class SuffixDrafter(_Handle):
    """Suffix drafter with frequency scoring (contexts up to ``max_depth``)."""
    _destroy = "sv_suffix_destroy"

    def __init__(self, max_depth: int = 8):
        super().__init__(_L().sv_suffix_create(int(max_depth)))
        self.max_depth = int(max_depth)     # the longest context tail a lookup can use

    def clear(self):
        _L().sv_suffix_clear(self._h)

    def append(self, problem_id: int, seq_id: int, tokens):
        t = _tok(tokens)
        if _L().sv_suffix_append(self._h, int(problem_id), int(seq_id), t.ctypes.data, t.size) != 0:
            raise ValueError("sv_suffix_append rejected its arguments")

    def draft(self, problem_id: int, context, k: int = 16) -> np.ndarray:
        c = _tail(context, self.max_depth)
        out = np.empty(max(int(k), 1), np.int32)
        n = _L().sv_suffix_draft(self._h, int(problem_id), c.ctypes.data, c.size, int(k), out.ctypes.data)
        if n < 0:
            raise ValueError("sv_suffix_draft rejected its arguments")
        return out[:n].copy()

    def draft_batch_flat(self, problem_ids, flat, offsets, k_max: int, max_lens=None, n_threads: int = 0):
        """Batched drafting on one flat context buffer, as
        NgramDrafter.draft_batch_flat."""
        return _draft_batch_flat(_L().sv_suffix_draft_batch, self._h, problem_ids, flat, offsets, k_max, max_lens,
                                 n_threads)

    def draft_batch(self, problem_ids, contexts, k_max: int, max_lens=None, n_threads: int = 0):
        """Batched drafting, as NgramDrafter.draft_batch."""
        return _draft_batch(_L().sv_suffix_draft_batch, self._h, problem_ids, contexts, k_max, max_lens, n_threads,
                            self.max_depth)

    def candidates(self, problem_id: int, context, f: int) -> np.ndarray:
        c = _tail(context, self.max_depth)
        out = np.empty(max(int(f), 1), np.int32)
        n = _L().sv_suffix_candidates(self._h, int(problem_id), c.ctypes.data, c.size, int(f), out.ctypes.data)
        if n < 0:
            raise ValueError("sv_suffix_candidates rejected its arguments")
        return out[:n].copy()


class PrefetchBudget(_Handle):
    """Fan-out prefetch budget over verification outcomes (j, rank of b)."""
    _destroy = "sv_prefetch_destroy"

    def __init__(self, k: int, fmax: int = 16, window: int = 256):
        super().__init__(_L().sv_prefetch_create(int(k), int(fmax), int(window)))
        self.k, self.fmax = int(k), int(fmax)

    def observe(self, j: int, b_rank: int):
        if _L().sv_prefetch_observe(self._h, int(j), int(b_rank)) != 0:
            raise ValueError("sv_prefetch_observe rejected its arguments")

    def estimates(self):
        P = np.empty(self.k + 1, np.float64)
        cov = np.empty((self.k + 1, self.fmax + 1), np.float64)
        n = _L().sv_prefetch_estimates(self._h, P.ctypes.data, cov.ctypes.data)
        return int(n), P, cov

    def allocate(self, budget: int = 16):
        f = np.empty(self.k + 1, np.int32)
        cov = _L().sv_prefetch_allocate(self._h, int(budget), f.ctypes.data)
        return f, float(cov)


class FanoutPrefetcher:
    """The fan-out pipeline around one NgramDrafter: while a request's draft
    is being verified, ``prepare`` spends the budget (PrefetchBudget over the
    recent outcomes) and drafts ahead for the outcomes it covers;
    ``next_draft`` then serves the draft for the actual outcome (j, b) from
    them (a hit) or drafts synchronously (a miss), and feeds the rank of b
    among branch j's candidates back into the budget's window.  Drafts are
    identical either way: prefetching only moves work off the critical path.
    Requests are told apart by a caller-chosen key."""

    def __init__(self, drafter: NgramDrafter, k: int = 16, budget: int = 16, fmax: int = 16, window: int = 256):
        self.drafter, self.k, self.n_budget, self.fmax = drafter, int(k), int(budget), int(fmax)
        self.budget = PrefetchBudget(self.k, self.fmax, window)
        self.hits = self.misses = 0
        self._pending = {}

    def prepare(self, key, prompt_id: int, context, draft) -> float:
        """Prefetch for request ``key`` (draft of at most k ids); returns the
        expected hit rate the allocation predicts."""
        # a lookup reads at most the last max_n tokens of its context, and a
        # branch only appends tokens to this one: its tail lies within ours
        ctx = [int(x) for x in _tail(context, self.drafter.max_n)]
        d = [int(x) for x in draft]
        if len(d) > self.k:
            raise ValueError(f"draft of {len(d)} ids, the prefetcher was built for k = {self.k}")
        f, coverage = self.budget.allocate(self.n_budget)
        pre = self.drafter.prefetch(prompt_id, ctx, d, f[:len(d) + 1], self.k)
        self._pending[key] = (prompt_id, ctx, d, pre)
        return coverage

    def next_draft(self, key, j: int, b: int):
        """The next draft of request ``key`` after outcome (j, b), and
        whether it came from the prefetch."""
        prompt_id, ctx, d, pre = self._pending.pop(key)
        branch = ctx + d[:j]
        ranked = [int(x) for x in self.drafter.candidates(prompt_id, branch, self.fmax)]
        self.budget.observe(j, ranked.index(b) if b in ranked else -1)
        got = pre.get((int(j), int(b)))
        if got is not None:
            self.hits += 1
            return got, True
        self.misses += 1
        return self.drafter.draft(prompt_id, branch + [int(b)], self.k), False


class DraftLengthController(_Handle):
    """Adaptive draft length over ascending candidate lengths."""
    _destroy = "sv_draft_len_destroy"

    def __init__(self, lengths=(5, 7, 9, 11), up_frac: float = 0.7, down_frac: float = 0.4, patience: int = 2):
        ls = _tok(lengths)
        super().__init__(_L().sv_draft_len_create(ls.ctypes.data, ls.size, float(up_frac), float(down_frac),
                                                  int(patience)))

    @property
    def current(self) -> int:
        return int(_L().sv_draft_len_current(self._h))

    def update(self, block_efficiency: float) -> int:
        return int(_L().sv_draft_len_update(self._h, float(block_efficiency)))


def block_efficiency(accept_len) -> float:
    a = _tok(accept_len)
    return float(_L().sv_block_efficiency(a.ctypes.data, a.size))


def spec_switch(state: list, predicted_speedup: float, threshold: float = 1.05) -> int:
    """``state`` is a one-element list holding the latch (0 at batch start)."""
    s = ctypes.c_int32(int(state[0]))
    r = _L().sv_spec_switch(ctypes.byref(s), float(predicted_speedup), float(threshold))
    state[0] = int(s.value)
    return int(r)


def length_classes(predicted_len, budgets=(0, 8, 16)):
    x = np.ascontiguousarray(np.asarray(predicted_len, np.float64).reshape(-1))
    b = np.ascontiguousarray(np.asarray(budgets, np.int32).reshape(3))
    cls = np.empty(x.size, np.int32)
    bud = np.empty(x.size, np.int32)
    if _L().sv_length_classes(x.ctypes.data, x.size, b.ctypes.data, cls.ctypes.data, bud.ctypes.data) != 0:
        raise ValueError("sv_length_classes rejected its arguments")
    return cls, bud


def interleave_ranks(predicted_len, world_size: int):
    x = np.ascontiguousarray(np.asarray(predicted_len, np.float64).reshape(-1))
    r = np.empty(x.size, np.int32)
    if _L().sv_interleave_ranks(x.ctypes.data, x.size, int(world_size), r.ctypes.data) != 0:
        raise ValueError("sv_interleave_ranks rejected its arguments")
    return r


# ---------------------------------------------------------------------------
# roofline predictor behind the speculation switch

class Arch(ctypes.Structure):
    """sv_arch: the decoder shape the roofline counts work from."""
    _fields_ = [("params", ctypes.c_double), ("weight_bytes", ctypes.c_double), ("layers", ctypes.c_int32),
                ("width", ctypes.c_int32), ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("kv_bytes", ctypes.c_double)]


class Roofline(ctypes.Structure):
    """sv_roofline: calibrated compute rate, bandwidth and per-step overhead."""
    _fields_ = [("flops_per_s", ctypes.c_double), ("bytes_per_s", ctypes.c_double),
                ("overhead_s", ctypes.c_double)]


def roofline_work(arch: Arch, B, q, n):
    """(flops, bytes) of one step over B sequences, q new tokens, n cached."""
    f, b = ctypes.c_double(), ctypes.c_double()
    if _L().sv_roofline_work(ctypes.byref(arch), float(B), float(q), float(n), ctypes.byref(f), ctypes.byref(b)):
        raise ValueError("sv_roofline_work rejected its arguments")
    return f.value, b.value


def roofline_time(arch: Arch, roof: Roofline, B, q, n) -> float:
    return float(_L().sv_roofline_time(ctypes.byref(arch), ctypes.byref(roof), float(B), float(q), float(n)))


def roofline_fit(arch: Arch, B, q, n, seconds):
    """Calibrate on measured steps; returns (Roofline, rms relative error)."""
    cols = [np.ascontiguousarray(np.asarray(x, dtype=np.float64).reshape(-1)) for x in (B, q, n, seconds)]
    m = cols[0].size
    if any(c.size != m for c in cols):
        raise ValueError("B, q, n and seconds must have the same length")
    out, rms = Roofline(), ctypes.c_double()
    if _L().sv_roofline_fit(ctypes.byref(arch), m, *(c.ctypes.data for c in cols), ctypes.byref(out),
                            ctypes.byref(rms)):
        raise ValueError("sv_roofline_fit rejected its arguments")
    return out, rms.value


def spec_speedup(target: Arch, rt: Roofline, draft: Arch, rd: Roofline, B, k: int, alpha: float, n) -> float:
    """Predicted speedup of speculative decoding over plain decoding."""
    return float(_L().sv_spec_speedup(ctypes.byref(target), ctypes.byref(rt), ctypes.byref(draft), ctypes.byref(rd),
                                      float(B), int(k), float(alpha), float(n)))
