"""Thin Python binding of liblosa.so (include/losa.h).

Argument marshalling only: tensors supply device memory, the current torch
CUDA stream supplies the stream, and every step of the computation runs in
the library's kernels. There is no fallback: if liblosa.so is missing or
fails to load, importing this package raises.

    import block_sparse_attention_losa_b200 as losa
    o, lse, mass = losa.dense_mass(q, k, v, L, block)        # construction step
    pat = losa.select(mass, block, tau=0.99)                   # frozen pattern
    o2, lse2 = losa.sparse_attn(q2, k2, v2, L, pat)            # every later step
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblosa.so")

LOSA_BF16, LOSA_FP32 = 0, 1
LOSA_OK = 0
STATUS = {0: "LOSA_OK", -1: "LOSA_ERR_ARG", -2: "LOSA_ERR_CUDA", -3: "LOSA_ERR_NOMEM",
          -4: "LOSA_ERR_TIMEOUT", -5: "LOSA_ERR_MASS", -6: "LOSA_ERR_UNSUPPORTED"}

# Every symbol include/losa.h declares.
EXPORTS = ("losa_dense_mass", "losa_select", "losa_dense_mass_select", "losa_pattern_info",
           "losa_pattern_export",
           "losa_pattern_import", "losa_select_noalloc", "losa_sparse_attn", "losa_free",
           "losa_check_status", "losa_selftest_wait", "losa_set_wait_limit", "losa_exp2_eval",
           "losa_strerror", "losa_version")
NOALLOC_MAX_ROWS = 65536  # LOSA_NOALLOC_MAX_ROWS


class LosaError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} "
                         f"({_lib.losa_strerror(status).decode()})")


class PatternView(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("n_blocks", ctypes.c_int),
                ("block", ctypes.c_int), ("nnz", ctypes.c_int64),
                ("row_ptr", ctypes.c_void_p), ("col_idx", ctypes.c_void_p),
                ("retained_fx", ctypes.c_void_p), ("total_fx", ctypes.c_void_p),
                ("n_tiles", ctypes.c_int64), ("tile_entries", ctypes.c_int64),
                ("tile_ptr", ctypes.c_void_p), ("tile_entry", ctypes.c_void_p),
                ("tile_order", ctypes.c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python block_sparse_attention_losa_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_double
    lib.losa_dense_mass.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32,
                                    vp, i32, vp, vp, vp]
    lib.losa_dense_mass.restype = i32
    lib.losa_select.argtypes = [vp, i32, i32, i32, i32, f64, ctypes.POINTER(vp), vp]
    lib.losa_select.restype = i32
    lib.losa_dense_mass_select.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32,
                                           f64, vp, i32, vp, vp, ctypes.POINTER(vp), vp]
    lib.losa_dense_mass_select.restype = i32
    lib.losa_pattern_info.argtypes = [vp, ctypes.POINTER(PatternView)]
    lib.losa_pattern_info.restype = i32
    lib.losa_pattern_export.argtypes = [vp] * 9
    lib.losa_pattern_export.restype = i32
    lib.losa_pattern_import.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32,
                                        ctypes.POINTER(vp), vp]
    lib.losa_pattern_import.restype = i32
    i64 = ctypes.c_int64
    lib.losa_select_noalloc.argtypes = [vp, i32, i32, i32, f64, vp, vp, i64, vp, vp, vp]
    lib.losa_select_noalloc.restype = i32
    lib.losa_sparse_attn.argtypes = [vp, vp, vp, i32, i32, i32, f32, vp, vp, i32, vp, vp]
    lib.losa_sparse_attn.restype = i32
    lib.losa_free.argtypes = [vp]
    lib.losa_free.restype = None
    lib.losa_check_status.argtypes = [vp]
    lib.losa_check_status.restype = i32
    lib.losa_selftest_wait.argtypes = [i64, vp]
    lib.losa_selftest_wait.restype = i32
    lib.losa_set_wait_limit.argtypes = [i64]
    lib.losa_set_wait_limit.restype = i32
    lib.losa_exp2_eval.argtypes = [vp, vp, i64, vp]
    lib.losa_exp2_eval.restype = i32
    lib.losa_strerror.argtypes = [i32]
    lib.losa_strerror.restype = ctypes.c_char_p
    lib.losa_version.argtypes = []
    lib.losa_version.restype = ctypes.c_char_p
    return lib


_lib = _load()


def lib():
    return _lib


def _check(fn, status):
    if status != LOSA_OK:
        raise LosaError(fn, status)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LOSA_BF16
    if t.dtype == torch.float32:
        return LOSA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check_qkv(q, k, v):
    for t in (q, k, v):
        if not (t.is_cuda and t.is_contiguous() and t.dim() == 4):
            raise ValueError("q, k, v must be contiguous CUDA tensors [B, H, L_pad, d]")
    if not (q.shape == k.shape == v.shape and q.dtype == k.dtype == v.dtype):
        raise ValueError("q, k, v must share shape and dtype")


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def dense_mass(q, k, v, L, block, scale=None, out_dtype=torch.float32, o=None, lse=None,
               mass=None, stream=None):
    """Construction step: (o, lse, mass) with mass [B, H, n, n], n = L_pad/block."""
    _check_qkv(q, k, v)
    B, H, Lp, d = q.shape
    n = Lp // block
    scale = default_scale(d) if scale is None else scale
    dev = q.device
    if o is None:
        o = torch.empty(B, H, Lp, d, device=dev, dtype=out_dtype)
    if lse is None:
        lse = torch.empty(B, H, Lp, device=dev, dtype=torch.float32)
    if mass is None:
        mass = torch.empty(B, H, n, n, device=dev, dtype=torch.float32)
    st = _lib.losa_dense_mass(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), B, H,
                              int(L), Lp, d, int(block), float(scale), o.data_ptr(),
                              _dtype_code(o), lse.data_ptr(), mass.data_ptr(), _stream(stream))
    _check("losa_dense_mass", st)
    return o, lse, mass


class Pattern:
    """A frozen block pattern owned by the library (freed on close / GC)."""

    def __init__(self, handle, device):
        self._h = handle
        self.device = device
        v = PatternView()
        _check("losa_pattern_info", _lib.losa_pattern_info(handle, ctypes.byref(v)))
        self.B, self.H, self.n_blocks, self.block = v.B, v.H, v.n_blocks, v.block
        self.nnz, self.n_tiles, self.tile_entries = v.nnz, v.n_tiles, v.tile_entries
        self._view = v

    @property
    def handle(self):
        if self._h is None:
            raise ValueError("pattern was freed")
        return self._h

    def close(self):
        if self._h is not None:
            _lib.losa_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def rows(self):
        return self.B * self.H * self.n_blocks

    def density(self):
        return self.nnz / float(self.rows * self.n_blocks)

    def export(self, device=None, stream=None):
        """Copies of the pattern arrays as torch tensors (on `device`,
        default the pattern's device; 'cpu' gives host copies)."""
        device = self.device if device is None else torch.device(device)
        pin = device.type == "cpu"
        sizes = dict(row_ptr=(self.rows + 1, torch.int32), col_idx=(self.nnz, torch.int32),
                     retained_fx=(self.rows, torch.int64), total_fx=(self.rows, torch.int64),
                     tile_ptr=(self.n_tiles + 1, torch.int32),
                     tile_entry=(self.tile_entries, torch.int32),
                     tile_order=(self.n_tiles, torch.int32))
        out = {k: torch.empty(int(n), dtype=dt, device=device, pin_memory=pin)
               for k, (n, dt) in sizes.items()}
        ptr = lambda t: t.data_ptr() if t.numel() else None
        st = _lib.losa_pattern_export(self.handle, *(ptr(out[k]) for k in sizes),
                                      _stream(stream))
        _check("losa_pattern_export", st)
        return out


def select(mass, block, tau=0.99, stream=None):
    """Selection step: a Pattern from a [B, H, n, n] fp32 mass map."""
    if not (mass.is_cuda and mass.is_contiguous() and mass.dtype == torch.float32
            and mass.dim() == 4 and mass.shape[2] == mass.shape[3]):
        raise ValueError("mass must be a contiguous fp32 CUDA tensor [B, H, n, n]")
    B, H, n, _ = mass.shape
    h = ctypes.c_void_p()
    st = _lib.losa_select(mass.data_ptr(), B, H, n, int(block), float(tau), ctypes.byref(h),
                          _stream(stream))
    _check("losa_select", st)
    return Pattern(h, mass.device)


def dense_mass_select(q, k, v, L, block, tau=0.99, scale=None, out_dtype=torch.float32,
                      o=None, lse=None, mass=None, stream=None):
    """Construction and selection in one call, the per-row cut fused into
    the construction kernel: (o, lse, mass, Pattern), each as dense_mass and
    select would give them."""
    _check_qkv(q, k, v)
    B, H, Lp, d = q.shape
    n = Lp // block
    scale = default_scale(d) if scale is None else scale
    dev = q.device
    if o is None:
        o = torch.empty(B, H, Lp, d, device=dev, dtype=out_dtype)
    if lse is None:
        lse = torch.empty(B, H, Lp, device=dev, dtype=torch.float32)
    if mass is None:
        mass = torch.empty(B, H, n, n, device=dev, dtype=torch.float32)
    h = ctypes.c_void_p()
    st = _lib.losa_dense_mass_select(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q),
                                     B, H, int(L), Lp, d, int(block), float(scale), float(tau),
                                     o.data_ptr(), _dtype_code(o), lse.data_ptr(),
                                     mass.data_ptr(), ctypes.byref(h), _stream(stream))
    _check("losa_dense_mass_select", st)
    return o, lse, mass, Pattern(h, dev)


def import_pattern(row_ptr, col_idx, B, H, n_blocks, block, retained_fx=None, total_fx=None,
                   device=None, stream=None):
    """A Pattern from a stored host CSR (e.g. Pattern.export('cpu') of an
    earlier selection). Arrays are converted to contiguous host int32/int64."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None \
        else torch.device(device)
    host = lambda t, dt: None if t is None else \
        torch.as_tensor(t).to("cpu", dtype=dt).contiguous()
    rp, ci = host(row_ptr, torch.int32), host(col_idx, torch.int32)
    rf, tf = host(retained_fx, torch.int64), host(total_fx, torch.int64)
    R = int(B) * int(H) * int(n_blocks)
    if rp.numel() != R + 1 or ci.numel() != int(rp[-1]) or \
            any(t is not None and t.numel() != R for t in (rf, tf)):
        raise ValueError("CSR array sizes do not match B * H * n_blocks")
    ptr = lambda t: None if t is None or t.numel() == 0 else t.data_ptr()
    h = ctypes.c_void_p()
    with torch.cuda.device(device):
        st = _lib.losa_pattern_import(ptr(rp), ptr(ci), ptr(rf), ptr(tf), int(B), int(H),
                                      int(n_blocks), int(block), ctypes.byref(h),
                                      _stream(stream))
    _check("losa_pattern_import", st)
    return Pattern(h, device)


def sparse_attn(q, k, v, L, pattern: Pattern, scale=None, out_dtype=torch.float32, o=None,
                lse=None, want_lse=True, stream=None):
    """Sparse step over a frozen pattern: (o, lse or None)."""
    _check_qkv(q, k, v)
    B, H, Lp, d = q.shape
    if (B, H, Lp) != (pattern.B, pattern.H, pattern.n_blocks * pattern.block):
        raise ValueError("q/k/v shape does not match the pattern")
    scale = default_scale(d) if scale is None else scale
    if o is None:
        o = torch.empty(B, H, Lp, d, device=q.device, dtype=out_dtype)
    if lse is None and want_lse:
        lse = torch.empty(B, H, Lp, device=q.device, dtype=torch.float32)
    st = _lib.losa_sparse_attn(q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q), d,
                               int(L), float(scale), pattern.handle, o.data_ptr(),
                               _dtype_code(o), lse.data_ptr() if lse is not None else None,
                               _stream(stream))
    _check("losa_sparse_attn", st)
    return o, lse


def exp2_eval(x, stream=None):
    """2^x with the kernels' FMA-pipe exponential (diagnostic)."""
    if not (x.is_cuda and x.is_contiguous() and x.dtype == torch.float32):
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    _check("losa_exp2_eval", _lib.losa_exp2_eval(x.data_ptr(), y.data_ptr(), x.numel(),
                                                 _stream(stream)))
    return y


def check_status(stream=None):
    """Synchronises the stream and raises if a kernel reported a timeout."""
    _check("losa_check_status", _lib.losa_check_status(_stream(stream)))


def set_wait_limit(cycles: int = 0):
    """Wait limit of later attention launches in SM cycles (0 = default,
    about 2 s); a diagnostic of the kernels' failure path."""
    _check("losa_set_wait_limit", _lib.losa_set_wait_limit(int(cycles)))


def version() -> str:
    return _lib.losa_version().decode()
