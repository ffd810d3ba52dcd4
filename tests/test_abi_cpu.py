"""The C-ABI library on a machine without a GPU: it builds, loads, exports
every symbol include/*.h declares, and rejects bad arguments on the host
before any CUDA call.  No kernel is launched here."""
import ctypes
import re
from pathlib import Path

import pytest

import speculative_decoding_verification_92_b200 as sv
from speculative_decoding_verification_92_b200 import _Options, _Shape, Status

ROOT = Path(__file__).resolve().parents[1]
FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails before touching it


def declared_symbols():
    names = []
    for h in sorted((ROOT / "include").glob("*.h")):
        text = h.read_text()
        names += re.findall(r"SV_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_library_exports_every_declared_symbol():
    lib = sv.library()
    names = declared_symbols()
    assert len(names) >= 8, names
    for name in names:
        assert hasattr(lib, name), f"{name} is declared in include/ but not exported"
    assert sv.abi_version() == 3


def test_status_strings():
    lib = sv.library()
    for code in Status:
        s = lib.spec_verify_status_string(int(code))
        assert isinstance(s, bytes) and len(s) > 0
    assert lib.spec_verify_status_string(99) == b"unknown status"


PIECE_BYTES = 16384


def a256(n):
    return (n + 255) // 256 * 256


@pytest.mark.parametrize("B,k,V,dt", [(64, 8, 151936, sv.BF16), (256, 12, 128256, sv.F32),
                                      (4, 4, 1000, sv.F32), (3, 0, 5, sv.BF16), (0, 3, 100, sv.F32)])
def test_workspace_bytes(B, k, V, dt):
    """Rows are cut into 16 KiB pieces (P per row); the workspace holds one
    8-byte partial per (request, row slot, piece), the control words (two
    queue lengths and one piece counter per row-statistics launch of up to
    4096 requests), two queues of 48-byte draw records, one
    loss mark per request and 32 segment sums per (request, piece)."""
    es = 2 if dt == sv.BF16 else 4
    P = -(-V * es // PIECE_BYTES)
    ctrl = 4 * (2 + -(-B // 4096))
    want = (a256(8 * B * (2 * k + 1) * P) + a256(ctrl) + 2 * a256(48 * B) + a256(4 * B) + a256(4 * 32 * B * P))
    assert sv.workspace_bytes(B, k, V, dt) == want


def test_workspace_bytes_invalid_shape():
    lib = sv.library()
    assert lib.spec_verify_workspace_bytes(None) == 0
    assert sv.workspace_bytes(4, 4, 0, sv.F32) == 0
    assert sv.workspace_bytes(4, -1, 10, sv.F32) == 0
    assert sv.workspace_bytes(4, 4, 10, 9) == 0
    assert sv.workspace_bytes(4, 4, 10, sv.F32, row_stride=5) == 0


def call(shape=None, target=FAKE, draft=None, tokens=FAKE, lens=None, uniforms=FAKE, T=1.0, greedy=0,
         out_len=FAKE, out_tok=FAKE, ws=FAKE, ws_bytes=1 << 30, opts=None):
    lib = sv.library()
    if shape is None:
        shape = _Shape(4, 4, 1000, sv.F32, 0)
    return lib.spec_verify_ex(ctypes.byref(shape) if shape is not False else None, target, draft, tokens, lens,
                              uniforms, T, greedy, out_len, out_tok, ws, ws_bytes, None,
                              ctypes.byref(opts) if opts is not None else None)


@pytest.mark.parametrize("kwargs,want", [
    (dict(shape=False), Status.EINVAL),
    (dict(shape=_Shape(4, 4, 0, sv.F32, 0)), Status.EINVAL),
    (dict(shape=_Shape(-1, 4, 10, sv.F32, 0)), Status.EINVAL),
    (dict(shape=_Shape(4, -2, 10, sv.F32, 0)), Status.EINVAL),
    (dict(shape=_Shape(4, 4, 10, sv.F32, 9)), Status.EINVAL),
    (dict(shape=_Shape(4, 4, 10, 5, 0)), Status.EUNSUPPORTED),
    (dict(shape=_Shape(4, sv.MAX_K + 1, 10, sv.F32, 0)), Status.EUNSUPPORTED),
    (dict(shape=_Shape(4, 4, sv.MAX_V + 1, sv.F32, 0)), Status.EUNSUPPORTED),
    (dict(target=None), Status.EINVAL),
    (dict(tokens=None), Status.EINVAL),
    (dict(out_len=None), Status.EINVAL),
    (dict(out_tok=None), Status.EINVAL),
    (dict(uniforms=None), Status.EINVAL),
    (dict(T=0.0), Status.EINVAL),
    (dict(T=-1.0), Status.EINVAL),
    (dict(T=float("nan")), Status.EINVAL),
    (dict(T=float("inf")), Status.EINVAL),
    (dict(ws=None), Status.EINVAL),
    (dict(ws_bytes=8), Status.EINVAL),
    (dict(ws=FAKE + 4), Status.EINVAL),
])
def test_argument_errors_before_any_launch(kwargs, want):
    assert call(**kwargs) == want


def test_bad_options():
    o = _Options()
    o.reserved[3] = 1
    assert call(opts=o) == Status.EINVAL
    for kernel in (4, 7, -1):               # only AUTO, TMA, VEC16 and SCALAR exist
        o = _Options()
        o.stats_kernel = kernel
        assert call(opts=o) == Status.EINVAL
    o = _Options()
    o.wait_timeout_us = -5
    assert call(opts=o) == Status.EINVAL
    for path in (3, -1):                    # only AUTO, QUEUE and CLUSTER exist
        o = _Options()
        o.draw_path = path
        assert call(opts=o) == Status.EINVAL
    for r in (-1, 5):                      # names no request of the B = 4 batch
        o = _Options()
        o.lost_copy_request = r
        assert call(opts=o) == Status.EINVAL
        o = _Options()
        o.lost_draw_request = r
        assert call(opts=o) == Status.EINVAL


def test_greedy_needs_no_uniforms_or_temperature_and_empty_batch_is_ok():
    # greedy: uniforms NULL and T = 0 pass validation; with B = 0 nothing is launched
    assert call(shape=_Shape(0, 4, 1000, sv.F32, 0), uniforms=None, T=0.0, greedy=1) == Status.OK
    assert call(shape=_Shape(0, 4, 1000, sv.F32, 0)) == Status.OK


def test_valid_call_without_gpu_reports_cuda_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert call() == Status.ECUDA


def test_stats_and_host_entry_points_validate():
    lib = sv.library()
    shape = _Shape(4, 4, 1000, sv.F32, 0)
    # stats: missing lse output
    assert lib.spec_verify_stats(ctypes.byref(shape), FAKE, None, FAKE, None, 1.0, None, None, None, None,
                                 FAKE, 1 << 20, None, None) == Status.EINVAL
    # host form: staging too small
    n = lib.spec_verify_host_staging_bytes(ctypes.byref(shape), 1, 0)
    assert n >= 4 * 5 * 1000 * 4 + 4 * 4 * 1000 * 4
    assert lib.spec_verify_host(ctypes.byref(shape), FAKE, FAKE, FAKE, None, FAKE, 1.0, 0, FAKE, FAKE,
                                FAKE, n - 1, FAKE, 1 << 20, None) == Status.EINVAL


def test_python_binding_rejects_host_tensors():
    import torch
    t = torch.zeros(2, 3, 10)
    with pytest.raises(ValueError):
        sv.spec_verify(t, None, torch.zeros(2, 2, dtype=torch.int32), None, torch.zeros(2, 3))


@pytest.mark.parametrize("bad,msg", [
    (dict(tokens=(3, 3)), "draft_tokens must have shape"),
    (dict(lens=(4,)), "draft_lens must have shape"),
    (dict(uniforms=(3, 4)), "uniforms must have shape"),
    (dict(out_tok=(3, 4)), "out_tokens must have shape"),
    (dict(out_len=(2,)), "out_accept_len must have shape"),
])
def test_python_binding_checks_shapes_before_any_call(bad, msg):
    # the library reads exactly B*k ids, B lengths and B*(k+1) uniforms
    # through raw pointers, so a wrongly shaped tensor must never reach it
    import torch
    B, k, V = 3, 4, 64
    shapes = dict(tokens=(B, k), lens=(B,), uniforms=(B, k + 1), out_len=(B,), out_tok=(B, k + 1))
    shapes.update(bad)
    i32 = lambda key: torch.zeros(shapes[key], dtype=torch.int32)
    with pytest.raises(ValueError, match=msg):
        sv.spec_verify(torch.zeros(B, k + 1, V), torch.zeros(B, k, V), i32("tokens"), i32("lens"),
                       torch.zeros(shapes["uniforms"]), out=(i32("out_len"), i32("out_tok")))


def test_size_limits_match_the_header():
    text = (Path(__file__).resolve().parents[1] / "include" / "spec_verify.h").read_text()
    assert int(re.search(r"#define SV_MAX_K (\d+)", text).group(1)) == sv.MAX_K
    assert int(re.search(r"#define SV_MAX_V (\d+)", text).group(1)) == sv.MAX_V
    lib = sv.library()
    for dt in (sv.F32, sv.BF16):
        assert lib.spec_verify_workspace_bytes(ctypes.byref(_Shape(3, sv.MAX_K, sv.MAX_V, dt, 0))) > 0
        assert lib.spec_verify_workspace_bytes(ctypes.byref(_Shape(3, 2, sv.MAX_V + 1, dt, 0))) == 0


def test_auto_draw_path_rejects_bad_shapes_and_needs_a_gpu():
    lib = sv.library()
    assert lib.spec_verify_auto_draw_path(ctypes.byref(_Shape(4, 4, 0, sv.F32, 0))) == -1
    assert lib.spec_verify_auto_draw_path(ctypes.byref(_Shape(-1, 4, 10, sv.F32, 0))) == -1
    import torch
    if not torch.cuda.is_available():
        assert lib.spec_verify_auto_draw_path(ctypes.byref(_Shape(4, 4, 1000, sv.F32, 0))) == -1
