"""CPU oracle for speculative-sampling verification (test infrastructure only).

This package is used by ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference arm of ``bench.py``; nothing on the product path
imports it.  The arithmetic lives in ``oracle.c`` (plain C, double precision,
sequential loops); this module only builds it with gcc and marshals numpy
arrays through ctypes.

Input conventions mirror the library under test: logits are float32 arrays or
bfloat16 bit patterns stored as uint16 arrays, shaped ``[B, k_max+1, row_stride]``
(target) and ``[B, k_max, row_stride]`` (draft, or ``None`` for one-hot q).
Uniforms are float32 ``[B, k_max+1]`` (converted exactly to double here) or
float64 for probing the rule at full double resolution.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "oracle.c"
_LIB = _HERE / "liboracle.so"

FLAG_ACCEPT_TIE = 1
FLAG_DRAW_TIE = 2
FLAG_INVALID = 4
FLAG_ZERO_RESIDUAL = 8
FLAG_DRAW_FALLBACK = 16
FLAG_NEAR_TIE = FLAG_ACCEPT_TIE | FLAG_DRAW_TIE

F32 = 0
BF16 = 1


def build(src: Path = _SRC, out: Path = _LIB, extra_flags=()) -> Path:
    """Compile ``oracle.c`` into a shared library with gcc (IEEE semantics:
    no fast-math, so sums stay sequential)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
           *extra_flags, "-o", str(out), str(src), "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(src: Path, out: Path) -> bool:
    return not out.exists() or out.stat().st_mtime < src.stat().st_mtime


class Oracle:
    """ctypes front-end of one compiled copy of ``oracle.c``."""

    def __init__(self, lib_path: os.PathLike | None = None):
        if lib_path is None:
            if _needs_build(_SRC, _LIB):
                build()
            lib_path = _LIB
        self.lib_path = Path(lib_path)
        self._lib = ctypes.CDLL(str(self.lib_path))
        f = self._lib.oracle_spec_verify
        i64, i32, vp, dbl = ctypes.c_int64, ctypes.c_int32, ctypes.c_void_p, ctypes.c_double
        f.argtypes = [i64, i32, i64, i32, i64, i64, i64, vp, vp, vp, vp, vp,
                      dbl, i32, vp, vp, vp, vp, vp, vp, vp]
        f.restype = ctypes.c_int
        self._f = f
        g = self._lib.oracle_accept_sim
        g.argtypes = [i64, i32, i64, vp, vp, vp, vp, vp, dbl, vp, vp, vp, vp]
        g.restype = ctypes.c_int
        self._g = g

    def verify(self, target, draft, tokens, lens, uniforms, temperature=1.0,
               greedy=False, *, V=None, B=None, diag=False):
        """Run the rule on every request; returns a dict of numpy arrays:
        ``len`` [B], ``tokens`` [B, k_max+1], ``flags`` [B] and, with
        ``diag=True``, ``lse_t`` [B, k_max+1], ``lse_d``, ``p``, ``q`` [B, k_max]
        (natural-log lse; NaN where a row is not used).

        A leading dimension of 1 on ``target``/``draft`` with ``B`` given
        repeats the same logits for all B requests."""
        target = np.ascontiguousarray(target)
        if target.dtype == np.float32:
            dtype = F32
        elif target.dtype == np.uint16:
            dtype = BF16
        else:
            raise TypeError("target must be float32 or uint16 (bf16 bits)")
        nb, k1, row_stride = target.shape
        k_max = k1 - 1
        if B is None:
            B = nb
        if V is None:
            V = row_stride
        req_t = 0 if (nb == 1 and B != 1) else k1 * row_stride
        req_d = 0
        if draft is not None:
            draft = np.ascontiguousarray(draft)
            if draft.dtype != target.dtype:
                raise TypeError("draft dtype must match target dtype")
            if draft.shape[1:] != (k_max, row_stride):
                raise ValueError("draft must be [B, k_max, row_stride]")
            req_d = 0 if (draft.shape[0] == 1 and B != 1) else k_max * row_stride
        tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k_max)
        if lens is not None:
            lens = np.ascontiguousarray(lens, dtype=np.int32).reshape(B)
        if uniforms is not None:
            uniforms = np.ascontiguousarray(uniforms, dtype=np.float64).reshape(B, k1)
        out_len = np.empty(B, np.int32)
        out_tok = np.empty((B, k1), np.int32)
        out_flags = np.empty(B, np.int32)
        lse_t = lse_d = p = q = None
        if diag:
            lse_t = np.empty((B, k1), np.float64)
            lse_d = np.full((B, k_max), np.nan)
            p = np.empty((B, k_max), np.float64)
            q = np.empty((B, k_max), np.float64)

        def ptr(a):
            return None if a is None else a.ctypes.data

        rc = self._f(B, k_max, V, dtype, row_stride, req_t, req_d, ptr(target),
                     ptr(draft), ptr(tokens), ptr(lens), ptr(uniforms),
                     float(temperature), int(bool(greedy)), ptr(out_len),
                     ptr(out_tok), ptr(out_flags), ptr(lse_t), ptr(lse_d),
                     ptr(p), ptr(q))
        if rc != 0:
            raise ValueError("oracle_spec_verify rejected its arguments")
        out = {"len": out_len, "tokens": out_tok, "flags": out_flags}
        if diag:
            out.update(lse_t=lse_t, lse_d=lse_d, p=p, q=q)
        return out


    def accept_sim(self, p, q, tokens, lens, uniforms=None, decay=0.8, *, V):
        """Acceptance simulation from per-position probabilities ``p``, ``q``
        [B, k_max] (float64, e.g. ``verify(..., diag=True)``'s): returns
        ``a`` [B, k_max], ``e`` [B] and, with uniforms, ``j`` [B] and ``w``
        [B, k_max] (else None)."""
        p = np.ascontiguousarray(p, dtype=np.float64)
        q = np.ascontiguousarray(q, dtype=np.float64)
        B, k_max = p.shape
        tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k_max)
        if lens is not None:
            lens = np.ascontiguousarray(lens, dtype=np.int32).reshape(B)
        if uniforms is not None:
            uniforms = np.ascontiguousarray(uniforms, dtype=np.float64).reshape(B, k_max + 1)
        a = np.empty((B, k_max), np.float64)
        e = np.empty(B, np.float64)
        j = np.empty(B, np.int32) if uniforms is not None else None
        w = np.empty((B, k_max), np.float64) if uniforms is not None else None

        def ptr(x):
            return None if x is None else x.ctypes.data

        self._g(B, k_max, int(V), ptr(tokens), ptr(lens), ptr(p), ptr(q), ptr(uniforms), float(decay),
                ptr(a), ptr(e), ptr(j), ptr(w))
        return {"a": a, "e": e, "j": j, "w": w}


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from this directory's ``oracle.c``."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


def verify(*args, **kwargs):
    return default().verify(*args, **kwargs)


def accept_sim(*args, **kwargs):
    return default().accept_sim(*args, **kwargs)
