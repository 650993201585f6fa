"""The C ABI without a GPU: libmsda.so loads, exports every function that
include/msda.h declares, and rejects bad arguments on the host (status code
and message, nothing launched).  Device pointers here are fake addresses that
are never dereferenced: every call returns before any CUDA call is made."""
import ctypes
import os
import re

import pytest

import scale_deformable_attention_03_b200 as msda
from scale_deformable_attention_03_b200 import build as msda_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msda.h")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA = 0, 1, 2, 3, 4
FAKE = 0x7f0000000000  # a 256-byte aligned address, never dereferenced


@pytest.fixture(scope="module")
def L():
    msda_build.build()
    return msda.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("msda_forward", "msda_forward_fused", "msda_backward", "msda_workspace_size",
              "sca_compact_workspace_size", "sca_compact", "sca_forward", "sca_backward",
              "sca_rebatched_forward", "sca_camera_average", "sca_rebatched_backward",
              "sca_camera_average_linear",
              "sca_compact_no_alloc", "msda_linear", "msda_linear_timeouts",
              "sca_module_forward", "sca_backward_inputs", "tsa_reference_points", "tsa_forward", "sca_forward_query_major",
              "msda_linear_dropout", "msda_backward_deterministic", "tsa_backward",
              "sca_backward_deterministic", "sca_backward_full", "sca_backward_full_workspace_size", "msda_linear_test_withhold_load",
              "msda_status_string", "msda_last_error", "msda_version"):
        assert n in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), f"libmsda.so does not export {name}"


def test_header_compiles_as_c():
    import subprocess
    import tempfile
    with tempfile.TemporaryDirectory() as d:
        src = os.path.join(d, "t.c")
        open(src, "w").write('#include "msda.h"\nint main(void){return (int)MSDA_OK;}\n')
        subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                        "-c", src, "-o", os.path.join(d, "t.o")], check=True)


def test_status_strings(L):
    assert L.msda_status_string(OK) == b"success"
    for code in (INVALID, UNSUPPORTED, WORKSPACE, CUDA):
        assert L.msda_status_string(code) not in (b"success", b"unknown status")
    assert L.msda_status_string(99) == b"unknown status"
    assert L.msda_version() >= 10000


def _levels(shapes):
    import numpy as np
    s = np.asarray(shapes, dtype=np.int64).reshape(-1, 2)
    st = np.concatenate([[0], np.cumsum(s[:, 0] * s[:, 1])[:-1]]).astype(np.int64)
    return s, st


def _fwd(L, dims, shapes=((4, 4),), value=FAKE, vdt=0, loc=FAKE, w=FAKE, out=FAKE):
    s, st = _levels(shapes)
    p = ctypes.POINTER(ctypes.c_int64)
    return L.msda_forward(value, vdt, s.ctypes.data_as(p), st.ctypes.data_as(p), loc, w,
                          msda.Dims(*dims), out, None)


GOOD = (1, 1, 8, 16, 2, 1, 4, 1)  # B, Ncam, Nq, Nv, H, L, P, R


@pytest.mark.parametrize("dims,code,fragment", [
    ((1, 1, 8, 16, 2, 0, 4, 1), UNSUPPORTED, "L = 0"),
    ((1, 1, 8, 16, 2, 9, 4, 1), UNSUPPORTED, "L = 9"),
    ((1, 1, 8, 16, 2, 1, 17, 1), UNSUPPORTED, "P = 17"),
    ((1, 1, 8, 16, 2, 1, 4, 3), INVALID, "divide P"),
    ((1, 1, 8, 16, 0, 1, 4, 1), INVALID, "H (0)"),
    ((-1, 1, 8, 16, 2, 1, 4, 1), INVALID, "B (-1)"),
    ((1, 1, 8, 15, 2, 1, 4, 1), INVALID, "does not fit"),
    ((1, 1, 8, 2 ** 26, 2, 1, 4, 1), UNSUPPORTED, "32-bit"),
])
def test_forward_rejects_bad_sizes(L, dims, code, fragment):
    assert _fwd(L, dims) == code
    assert fragment in L.msda_last_error().decode()


def test_forward_rejects_bad_pointers(L):
    assert _fwd(L, GOOD, value=0) == INVALID
    assert _fwd(L, GOOD, value=FAKE + 4) == INVALID
    assert "16-byte" in L.msda_last_error().decode()
    assert _fwd(L, GOOD, loc=0) == INVALID
    assert _fwd(L, GOOD, loc=FAKE + 4) == INVALID
    assert _fwd(L, GOOD, out=FAKE + 8) == INVALID
    assert _fwd(L, GOOD, vdt=7) == INVALID
    assert _fwd(L, GOOD, shapes=((0, 4),)) == INVALID


def test_empty_problem_is_a_no_op(L):
    assert _fwd(L, (0, 1, 8, 16, 2, 1, 4, 1), loc=0, w=0, out=0) == OK
    assert _fwd(L, (1, 1, 0, 16, 2, 1, 4, 1), loc=0, w=0, out=0) == OK
    assert L.msda_last_error() == b""


def _sca_fwd(L, dims, ws, ws_bytes, shapes=((4, 4),)):
    s, st = _levels(shapes)
    p = ctypes.POINTER(ctypes.c_int64)
    return L.sca_forward(FAKE, 0, s.ctypes.data_as(p), st.ctypes.data_as(p), FAKE, FAKE, FAKE,
                         FAKE, msda.Dims(*dims), ws, ws_bytes, FAKE, None)


def test_sca_workspace_checks(L):
    dims = (1, 6, 100, 16, 2, 1, 4, 2)
    need = L.msda_workspace_size(msda.Dims(*dims))
    assert need > 6 * 100 * 64 * 4   # the rebatched rows dominate
    assert _sca_fwd(L, dims, 0, need) == WORKSPACE
    assert _sca_fwd(L, dims, FAKE, need - 1) == WORKSPACE
    assert _sca_fwd(L, dims, FAKE + 8, need) == WORKSPACE
    assert _sca_fwd(L, (1, 33, 100, 16, 2, 1, 4, 2), FAKE, need) == UNSUPPORTED
    assert _sca_fwd(L, (1, 0, 100, 16, 2, 1, 4, 2), FAKE, need) == UNSUPPORTED


def test_workspace_sizes_bevformer_base(L):
    d = msda.Dims(1, 6, 40000, 30825, 8, 4, 8, 4)
    rows = 6 * 40000 * 256 * 4
    lists = 2 * 6 * 40000 * 4 + 40000 * 4
    ws = L.msda_workspace_size(d)
    assert rows + lists <= ws <= rows + lists + 64 * 1024
    cws = L.sca_compact_workspace_size(d)
    assert 0 < cws <= 4096
    assert L.msda_workspace_size(msda.Dims(1, 0, 4, 4, 1, 1, 1, 1)) == 0


def test_compact_rejects_bad_arguments(L):
    d = msda.Dims(1, 6, 100, 1, 1, 1, 1, 4)
    n = L.sca_compact_workspace_size(d)
    assert L.sca_compact(FAKE, d, FAKE, n - 1, FAKE, FAKE, FAKE, FAKE, None) == WORKSPACE
    assert L.sca_compact(0, d, FAKE, n, FAKE, FAKE, FAKE, FAKE, None) == INVALID
    assert L.sca_compact(FAKE, msda.Dims(1, 6, 100, 1, 1, 1, 1, 0), FAKE, n, FAKE, FAKE, FAKE,
                         FAKE, None) == INVALID
    assert L.sca_compact(FAKE, msda.Dims(0, 6, 100, 1, 1, 1, 1, 4), 0, 0, 0, 0, 0, 0, None) == OK
    big = msda.Dims(64, 32, 100, 1, 1, 1, 1, 4)   # B * Ncam = 2048 > 1024
    assert L.sca_compact(FAKE, big, FAKE, 1 << 20, FAKE, FAKE, FAKE, FAKE, None) == UNSUPPORTED


def test_backward_rejects_bad_arguments(L):
    s, st = _levels(((4, 4),))
    p = ctypes.POINTER(ctypes.c_int64)
    args = lambda gv, gl: L.msda_backward(FAKE, 0, s.ctypes.data_as(p), st.ctypes.data_as(p),  # noqa: E731
                                          FAKE, FAKE, FAKE, msda.Dims(*GOOD), gv, gl, FAKE, None)
    assert args(0, FAKE) == INVALID
    assert args(FAKE + 4, FAKE) == INVALID
    assert args(FAKE, 0) == INVALID


def test_binding_raises_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(msda, "_lib", None)
    monkeypatch.setattr(msda, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(msda.MsdaError):
        msda.lib()


def test_linear_rejects_unsupported_shapes(L):
    f = L.msda_linear
    assert f(FAKE, FAKE, None, None, 128, 100, 256, 0, FAKE, None) == UNSUPPORTED   # N
    assert f(FAKE, FAKE, None, None, 128, 256, 320, 0, FAKE, None) == UNSUPPORTED   # K
    assert f(FAKE, FAKE, None, None, 128, 256, 96, 0, FAKE, None) == UNSUPPORTED    # K
    assert f(FAKE + 8, FAKE, None, None, 128, 256, 256, 0, FAKE, None) == INVALID   # alignment
    assert f(FAKE, FAKE, FAKE + 4, None, 128, 256, 256, 0, FAKE, None) == INVALID   # bias
    assert f(FAKE, FAKE, None, None, 128, 256, 256, 9, FAKE, None) == INVALID       # dtype
    assert f(0, 0, None, None, 0, 256, 256, 0, 0, None) == OK                        # empty


def test_tsa_reference_points_rejects_bad_arguments(L):
    f = L.tsa_reference_points
    assert f(FAKE, -1, 2, 200, 200, 0.512, 0.512, FAKE, None) == INVALID      # B
    assert f(FAKE, 1, 0, 200, 200, 0.512, 0.512, FAKE, None) == INVALID       # queues
    assert f(FAKE, 1, 2, 0, 200, 0.512, 0.512, FAKE, None) == INVALID         # empty grid
    assert f(FAKE, 1, 2, 200, 200, 0.0, 0.512, FAKE, None) == INVALID         # grid length
    assert f(FAKE, 1, 2, 200, 200, 0.512, float("nan"), FAKE, None) == INVALID
    assert f(FAKE, 1, 2, 200, 200, 0.512, 0.512, FAKE + 4, None) == INVALID   # alignment
    assert f(0, 1, 2, 200, 200, 0.512, 0.512, FAKE, None) == INVALID          # null
    assert f(0, 0, 2, 200, 200, 0.512, 0.512, 0, None) == OK                  # empty batch


def test_tsa_forward_rejects_bad_arguments(L):
    s, st = _levels(((4, 4),))
    p = ctypes.POINTER(ctypes.c_int64)
    call = lambda T, d, out=FAKE: L.tsa_forward(  # noqa: E731
        FAKE, 0, s.ctypes.data_as(p), st.ctypes.data_as(p), FAKE, FAKE, FAKE, T, d, out, None)
    assert call(0, msda.Dims(*GOOD)) == UNSUPPORTED
    assert call(5, msda.Dims(*GOOD)) == UNSUPPORTED
    assert call(2, msda.Dims(*GOOD), FAKE + 4) == INVALID
    assert call(2, msda.Dims(*GOOD), 0) == INVALID
    empty = list(GOOD)
    empty[0] = 0
    assert call(2, msda.Dims(*empty), 0) == OK


def test_sca_query_major_rejects_bad_arguments(L):
    s, st = _levels(((4, 4),))
    p = ctypes.POINTER(ctypes.c_int64)
    call = lambda d, out=FAKE, mask=FAKE: L.sca_forward_query_major(  # noqa: E731
        FAKE, 0, s.ctypes.data_as(p), st.ctypes.data_as(p), FAKE, mask, FAKE, FAKE, d, out, None)
    assert call(msda.Dims(1, 33, 8, 16, 2, 1, 4, 1)) == UNSUPPORTED   # Ncam > 32
    assert call(msda.Dims(1, 0, 8, 16, 2, 1, 4, 1)) == UNSUPPORTED    # no camera
    assert call(msda.Dims(1, 6, 8, 16, 2, 1, 4, 1), out=0) == INVALID
    assert call(msda.Dims(1, 6, 8, 16, 2, 1, 4, 1), mask=0) == INVALID
    assert call(msda.Dims(1, 6, 8, 16, 2, 1, 4, 1), out=FAKE + 8) == INVALID
    assert call(msda.Dims(1, 6, 0, 16, 2, 1, 4, 1), out=0) == OK       # nothing to do


def test_linear_dropout_rejects_bad_rates(L):
    f = L.msda_linear_dropout
    for p in (-0.1, 1.0, 1.5, float("nan")):
        assert f(FAKE, FAKE, None, None, 128, 256, 256, 0, FAKE, p, 0, None) == INVALID
    assert f(0, 0, None, None, 0, 256, 256, 0, 0, 0.2, 1, None) == OK   # empty


def test_deterministic_backward_workspace_checks(L):
    s, st = _levels(((4, 4),))
    p = ctypes.POINTER(ctypes.c_int64)
    d = msda.Dims(*GOOD)
    need = L.msda_backward_deterministic_workspace_size(d)
    assert need >= 1 * 16 * 2 * 32 * 8
    call = lambda ws, n: L.msda_backward_deterministic(  # noqa: E731
        FAKE, 0, s.ctypes.data_as(p), st.ctypes.data_as(p), FAKE, FAKE, FAKE, d, ws, n, FAKE,
        FAKE, FAKE, None)
    assert call(0, need) == WORKSPACE
    assert call(FAKE, need - 8) == WORKSPACE
    sd = msda.Dims(1, 6, 8, 16, 2, 1, 4, 1)
    assert L.sca_backward_deterministic_workspace_size(sd) >= 6 * 16 * 2 * 32 * 8
