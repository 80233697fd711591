"""The C-ABI library loads, exports every symbol include/losa.h declares, and
rejects bad arguments on the host (no device work, so no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "losa.h")


def _build():
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "losa_build", os.path.join(ROOT, "block_sparse_attention_losa_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def losa():
    _build()
    import block_sparse_attention_losa_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(losa_\w+)\s*\(", text)))


def test_header_declares_the_four_method_calls():
    names = declared_functions()
    for n in ("losa_dense_mass", "losa_select", "losa_sparse_attn", "losa_free"):
        assert n in names


def test_library_exports_every_declared_symbol(losa):
    lib = ctypes.CDLL(losa.LIB_PATH)
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"liblosa.so does not export {n}"
    assert sorted(losa.EXPORTS) == names


def test_strerror_and_version(losa):
    lib = losa.lib()
    assert lib.losa_strerror(0) == b"ok"
    for code in range(-6, 0):
        assert lib.losa_strerror(code) != b"unknown status"
    assert lib.losa_strerror(-99) == b"unknown status"
    assert re.fullmatch(rb"\d+\.\d+\.\d+", lib.losa_version())


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: the checks fail first


def _dense(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, in_dt=0, B=1, H=2, L=250, L_pad=256, d=64, block=32,
             scale=0.125, o=FAKE, out_dt=1, lse=FAKE, mass=FAKE, stream=None)
    a.update(kw)
    return lib.losa_dense_mass(a["q"], a["k"], a["v"], a["in_dt"], a["B"], a["H"], a["L"],
                               a["L_pad"], a["d"], a["block"], a["scale"], a["o"], a["out_dt"],
                               a["lse"], a["mass"], a["stream"])


@pytest.mark.parametrize("bad", [
    dict(q=None), dict(mass=None), dict(lse=None), dict(in_dt=7), dict(out_dt=-1),
    dict(B=0), dict(H=0), dict(L=0), dict(L=300), dict(L_pad=250, L=250),
    dict(L=200), dict(d=96), dict(block=16), dict(block=256), dict(scale=0.0),
    dict(scale=float("nan")), dict(scale=float("inf")), dict(L=70000, L_pad=70016, block=32),
    dict(B=300, H=300), dict(q=ctypes.c_void_p(0x10008)),
])
def test_dense_mass_rejects_bad_arguments(losa, bad):
    assert _dense(losa.lib(), **bad) == -1


def _dense_select(lib, tau=0.99, out=True, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, in_dt=0, B=1, H=2, L=250, L_pad=256, d=64, block=32,
             scale=0.125, o=FAKE, out_dt=1, lse=FAKE, mass=FAKE, stream=None)
    a.update(kw)
    h = ctypes.c_void_p(123)
    st = lib.losa_dense_mass_select(a["q"], a["k"], a["v"], a["in_dt"], a["B"], a["H"], a["L"],
                                    a["L_pad"], a["d"], a["block"], a["scale"], tau, a["o"],
                                    a["out_dt"], a["lse"], a["mass"],
                                    ctypes.byref(h) if out else None, a["stream"])
    return st, h.value


@pytest.mark.parametrize("bad", [
    dict(q=None), dict(mass=None), dict(lse=None), dict(o=None), dict(in_dt=7), dict(B=0),
    dict(L=300), dict(L=200), dict(d=96), dict(block=16), dict(scale=0.0),
    dict(L=70000, L_pad=70016, block=32), dict(B=300, H=300), dict(v=ctypes.c_void_p(0x10004)),
    dict(tau=0.0), dict(tau=1.5), dict(tau=float("nan")), dict(out=False),
])
def test_dense_mass_select_rejects_bad_arguments(losa, bad):
    """The fused call checks what losa_dense_mass and losa_select check
    (shapes, dtypes, alignment, tau in (0, 1], a place for the pattern) on
    the host, and leaves the pattern slot NULL when it refuses."""
    st, h = _dense_select(losa.lib(), **bad)
    assert st == -1
    if bad != dict(out=False):
        assert h is None


@pytest.mark.parametrize("tau", [0.0, -0.5, 1.0000001, 2.0, float("nan")])
def test_select_rejects_tau_outside_unit_interval(losa, tau):
    out = ctypes.c_void_p(123)
    st = losa.lib().losa_select(FAKE, 1, 2, 8, 32, tau, ctypes.byref(out), None)
    assert st == -1 and out.value is None


@pytest.mark.parametrize("shape", [(0, 2, 8, 32), (1, 0, 8, 32), (1, 2, 0, 32),
                                   (1, 2, 2048, 32), (1, 2, 8, 48)])
def test_select_rejects_bad_shapes(losa, shape):
    out = ctypes.c_void_p()
    B, H, n, b = shape
    assert losa.lib().losa_select(FAKE, B, H, n, b, 0.99, ctypes.byref(out), None) == -1


def test_null_handles(losa):
    lib = losa.lib()
    view = losa.PatternView()
    assert lib.losa_pattern_info(None, ctypes.byref(view)) == -1
    assert lib.losa_sparse_attn(FAKE, FAKE, FAKE, 0, 64, 10, 0.1, None, FAKE, 1, None, None) == -1
    assert lib.losa_pattern_export(None, None, None, None, None, None, None, None, None) == -1
    lib.losa_free(None)  # no-op


def _import(losa, row_ptr, col_idx, B=1, H=1, n=4, block=64):
    rp = (ctypes.c_int32 * len(row_ptr))(*row_ptr)
    ci = (ctypes.c_int32 * max(len(col_idx), 1))(*col_idx)
    out = ctypes.c_void_p(1)
    st = losa.lib().losa_pattern_import(rp, ci, None, None, B, H, n, block, ctypes.byref(out),
                                        None)
    assert out.value is None  # *out is cleared on every failure
    return st


# One head, n = 4 key blocks, so 4 CSR rows; each case breaks one rule.
@pytest.mark.parametrize("row_ptr,col_idx", [
    ([1, 2, 3, 4, 5], [0, 0, 0, 0, 0]),            # row_ptr[0] != 0
    ([0, 1, 1, 2, 3], [0, 1, 2]),                  # an empty row
    ([0, 5, 6, 7, 8], [0, 1, 2, 3, 3, 0, 0, 0]),   # a row longer than n
    ([0, 2, 3, 4, 5], [1, 0, 0, 0, 0]),            # columns not ascending
    ([0, 2, 3, 4, 5], [1, 1, 0, 0, 0]),            # a repeated column
    ([0, 1, 2, 3, 4], [0, 4, 0, 0]),               # a column >= n
    ([0, 1, 2, 3, 4], [0, -1, 0, 0]),              # a negative column
    ([0, 1, 2, 1, 4], [0, 1, 2, 3]),               # row_ptr decreasing
])
def test_pattern_import_rejects_invalid_csr(losa, row_ptr, col_idx):
    assert _import(losa, row_ptr, col_idx) == -1


def test_pattern_import_rejects_bad_shapes_and_nulls(losa):
    lib = losa.lib()
    out = ctypes.c_void_p()
    rp = (ctypes.c_int32 * 5)(0, 1, 2, 3, 4)
    ci = (ctypes.c_int32 * 4)(0, 1, 2, 3)
    assert lib.losa_pattern_import(None, ci, None, None, 1, 1, 4, 64, ctypes.byref(out), None) == -1
    assert lib.losa_pattern_import(rp, None, None, None, 1, 1, 4, 64, ctypes.byref(out), None) == -1
    assert lib.losa_pattern_import(rp, ci, None, None, 1, 1, 4, 64, None, None) == -1
    assert lib.losa_pattern_import(rp, ci, None, None, 1, 1, 4, 48, ctypes.byref(out), None) == -1
    assert lib.losa_pattern_import(rp, ci, None, None, 1, 1, 2048, 64, ctypes.byref(out),
                                   None) == -1
    assert lib.losa_pattern_import(rp, ci, None, None, 0, 1, 4, 64, ctypes.byref(out), None) == -1


def test_pattern_import_accepts_a_valid_csr_up_to_the_device_check(losa):
    import torch
    if torch.cuda.is_available():
        pytest.skip("device path covered by the GPU tests")
    # Valid (diagonal plus one neighbour): passes the host checks, then the
    # device check reports that no sm_100 GPU is present.
    assert _import(losa, [0, 2, 4, 6, 7], [0, 1, 0, 1, 2, 3, 3]) == -6


def test_process_settings_reject_values_out_of_range(losa):
    """losa_set_wait_limit takes 0 (the default) to 2^33 SM cycles; anything
    else is refused on the host and leaves the setting as it was."""
    lib = losa.lib()
    for bad in (-1, (1 << 33) + 1, -(1 << 40)):
        assert lib.losa_set_wait_limit(bad) == -1
    assert lib.losa_set_wait_limit(0) == 0
    assert lib.losa_selftest_wait(0, None) == -1


def test_select_noalloc_rejects_bad_arguments(losa):
    """Host-side checks of the allocation-free selection, before any device
    work: null buffers, sizes, tau, a negative capacity, and more rows than
    its fixed scratch holds."""
    lib = losa.lib()
    call = lambda *a: lib.losa_select_noalloc(*a, None)
    ok = (FAKE, 1, 2, 8, ctypes.c_double(0.99), FAKE, FAKE, ctypes.c_int64(16), FAKE, FAKE)
    for i in (0, 5, 6, 8, 9):  # each pointer argument set to NULL
        args = list(ok)
        args[i] = None
        assert call(*args) == -1
    for B, H, n in ((0, 2, 8), (1, 0, 8), (1, 2, 0), (1, 2, 2048), (1, 40, 2047)):
        assert call(FAKE, B, H, n, ctypes.c_double(0.99), FAKE, FAKE, ctypes.c_int64(16),
                    FAKE, FAKE) == -1
    for tau in (0.0, 1.5, float("nan")):
        assert call(FAKE, 1, 2, 8, ctypes.c_double(tau), FAKE, FAKE, ctypes.c_int64(16),
                    FAKE, FAKE) == -1
    assert call(FAKE, 1, 2, 8, ctypes.c_double(0.99), FAKE, FAKE, ctypes.c_int64(-1),
                FAKE, FAKE) == -1
