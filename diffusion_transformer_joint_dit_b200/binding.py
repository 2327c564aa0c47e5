"""ctypes binding of the jattn C-ABI (``include/jattn.h``).

Argument marshalling only: every function forwards to the symbol of the same
name in ``_lib/libjattn.so``, whose CUDA kernels do all of the work.  Tensor
arguments may be torch tensors (their ``data_ptr()`` is passed), plain
integer addresses or ``None`` (NULL).  ``stream`` may be a
``torch.cuda.Stream``, an integer ``cudaStream_t`` handle, or ``None`` for
torch's current stream on the current device.  A non-OK status raises
:class:`JattnError`.  The library is loaded on first use; if it is missing or
cannot be loaded the call raises: there is no fallback.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libjattn.so")

JATTN_OK = 0
JATTN_ERR_INVALID_ARG = 1
JATTN_ERR_UNSUPPORTED = 2
JATTN_ERR_MISALIGNED = 3
JATTN_ERR_CUDA = 4
JATTN_ERR_TIMEOUT = 5
JATTN_PROLOGUE_BF16 = 0
JATTN_PROLOGUE_FP8 = 1
JATTN_FP8_BLOCK = 64
JATTN_MAX_REF_GRIDS = 8
JATTN_SPARSE_QBLOCK = 256
JATTN_SPARSE_KBLOCK = 128

EXPORTED = ("jattn_prologue", "jattn_fwd_bf16", "jattn_fwd_fp8", "jattn_rope_table", "jattn_qkv_fused",
            "jattn_fp8_repair_select", "jattn_fp8_repair_apply", "jattn_sparse_select", "jattn_fwd_bf16_sparse",
            "jattn_status_string", "jattn_device_status", "jattn_selftest_wait_timeout",
            "jattn_last_cuda_error", "jattn_sparse_select_noalloc")


class JattnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} failed: {status_name(status)} ({status})"
        if status == JATTN_ERR_CUDA:
            msg += f" [{jattn_last_cuda_error()}]"
        super().__init__(msg)


class jattn_ref_grid(ctypes.Structure):
    _fields_ = [("h", ctypes.c_int), ("w", ctypes.c_int), ("row_offset", ctypes.c_int), ("col_offset", ctypes.c_int)]


class jattn_prologue_params(ctypes.Structure):
    _fields_ = [
        ("img_h", ctypes.c_int), ("img_w", ctypes.c_int),
        ("ref_h", ctypes.c_int), ("ref_w", ctypes.c_int),
        ("ref_row_offset", ctypes.c_int),
        ("rope_theta", ctypes.c_float), ("eps", ctypes.c_float),
        ("q_norm_w", ctypes.c_void_p), ("k_norm_w", ctypes.c_void_p),
        ("n_ref_grids", ctypes.c_int), ("ref_grids", ctypes.POINTER(jattn_ref_grid)),
    ]


class jattn_qkv_weights(ctypes.Structure):
    _fields_ = [
        ("w_qkv", ctypes.c_void_p * 2),
        ("q_norm_w", ctypes.c_void_p * 2),
        ("k_norm_w", ctypes.c_void_p * 2),
        ("eps", ctypes.c_float),
    ]


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int


def load_library():
    """Load ``libjattn.so`` (once) and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"jattn CUDA library not built: {LIB_PATH} is missing "
                           "(run `python -c 'import __graft_entry__ as g; g.build()'`)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.jattn_prologue.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                   ctypes.POINTER(jattn_prologue_params), _P]
    lib.jattn_prologue.restype = _I
    lib.jattn_fwd_bf16.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P]
    lib.jattn_fwd_bf16.restype = _I
    lib.jattn_fwd_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P]
    lib.jattn_fwd_fp8.restype = _I
    lib.jattn_rope_table.argtypes = [_P, _I, _I, _I, ctypes.POINTER(jattn_prologue_params), _P]
    lib.jattn_rope_table.restype = _I
    lib.jattn_qkv_fused.argtypes = [_P, ctypes.POINTER(jattn_qkv_weights), _P, _P, _P, _P,
                                    _I, _I, _I, _I, _I, _I, _I, _P]
    lib.jattn_qkv_fused.restype = _I
    lib.jattn_fp8_repair_select.argtypes = [_P, _P, _P, _P, _P, _P, ctypes.POINTER(jattn_prologue_params), _I,
                                            _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]
    lib.jattn_fp8_repair_select.restype = _I
    lib.jattn_fp8_repair_apply.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                                           _I, _I, _I, _I, _I, _I, ctypes.c_float, _P]
    lib.jattn_fp8_repair_apply.restype = _I
    lib.jattn_sparse_select.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                        ctypes.c_float, ctypes.c_float, _P]
    lib.jattn_sparse_select.restype = _I
    lib.jattn_fwd_bf16_sparse.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _P]
    lib.jattn_fwd_bf16_sparse.restype = _I
    lib.jattn_sparse_select_noalloc.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                                ctypes.c_float, ctypes.c_float, _P]
    lib.jattn_sparse_select_noalloc.restype = _I
    lib.jattn_status_string.argtypes = [_I]
    lib.jattn_status_string.restype = ctypes.c_char_p
    lib.jattn_device_status.argtypes = [_P]
    lib.jattn_device_status.restype = _I
    lib.jattn_selftest_wait_timeout.argtypes = [ctypes.c_longlong, _P]
    lib.jattn_selftest_wait_timeout.restype = _I
    lib.jattn_last_cuda_error.argtypes = []
    lib.jattn_last_cuda_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(fn: str, status: int) -> None:
    if status != JATTN_OK:
        raise JattnError(fn, status)


def status_name(status: int) -> str:
    return load_library().jattn_status_string(int(status)).decode()


def jattn_status_string(status: int) -> str:
    return status_name(status)


def make_prologue_params(img_h: int, img_w: int, ref_h: int = 0, ref_w: int = 0, ref_row_offset: int = 0,
                         rope_theta: float = 10000.0, eps: float = 1e-6, q_norm_w=None, k_norm_w=None,
                         ref_grids=None):
    """Prologue parameters.  ``ref_grids``: optional sequence of
    ``(h, w, row_offset, col_offset)``, one per reference image, in sequence
    order; it replaces ref_h / ref_w / ref_row_offset."""
    p = jattn_prologue_params(img_h, img_w, ref_h, ref_w, ref_row_offset, rope_theta, eps,
                              _ptr(q_norm_w), _ptr(k_norm_w), 0, None)
    if ref_grids:
        arr = (jattn_ref_grid * len(ref_grids))(*[jattn_ref_grid(*g) for g in ref_grids])
        p.n_ref_grids = len(ref_grids)
        p.ref_grids = ctypes.cast(arr, ctypes.POINTER(jattn_ref_grid))
        p._grids_keepalive = arr  # the host array must outlive the calls that read it
    return p


def jattn_prologue(q, k, v, q_out, k_out, v_out, q_scale, k_scale, v_scale,
                   B: int, H: int, N_txt: int, N_img: int, N_ref: int, d: int, mode: int,
                   params: jattn_prologue_params, stream=None, *, check: bool = True) -> int:
    st = load_library().jattn_prologue(
        _ptr(q), _ptr(k), _ptr(v), _ptr(q_out), _ptr(k_out), _ptr(v_out),
        _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
        B, H, N_txt, N_img, N_ref, d, mode,
        ctypes.byref(params) if params is not None else None, _stream(stream))
    if check:
        _check("jattn_prologue", st)
    return st


def jattn_fwd_bf16(q, k, v, o, lse, B: int, H: int, N_txt: int, N_img: int, N_ref: int, d: int,
                   softmax_scale: float, stream=None, *, check: bool = True) -> int:
    st = load_library().jattn_fwd_bf16(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                       B, H, N_txt, N_img, N_ref, d, softmax_scale, _stream(stream))
    if check:
        _check("jattn_fwd_bf16", st)
    return st


def jattn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B: int, H: int, N_txt: int, N_img: int,
                  N_ref: int, d: int, softmax_scale: float, stream=None, *, check: bool = True) -> int:
    st = load_library().jattn_fwd_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale),
                                      _ptr(v_scale), _ptr(o), _ptr(lse), B, H, N_txt, N_img, N_ref, d,
                                      softmax_scale, _stream(stream))
    if check:
        _check("jattn_fwd_fp8", st)
    return st


def make_qkv_weights(w_txt, w_img, q_norm_w=(None, None), k_norm_w=(None, None), eps: float = 1e-6):
    """jattn_qkv_weights from per-stream tensors (text, image + reference)."""
    wt = jattn_qkv_weights()
    wt.w_qkv[0], wt.w_qkv[1] = _ptr(w_txt), _ptr(w_img)
    wt.q_norm_w[0], wt.q_norm_w[1] = _ptr(q_norm_w[0]), _ptr(q_norm_w[1])
    wt.k_norm_w[0], wt.k_norm_w[1] = _ptr(k_norm_w[0]), _ptr(k_norm_w[1])
    wt.eps = eps
    return wt


def jattn_rope_table(table, N_txt: int, N_img: int, N_ref: int, params: jattn_prologue_params, stream=None, *,
                     check: bool = True) -> int:
    st = load_library().jattn_rope_table(_ptr(table), N_txt, N_img, N_ref,
                                         ctypes.byref(params) if params is not None else None, _stream(stream))
    if check:
        _check("jattn_rope_table", st)
    return st


def jattn_qkv_fused(x, weights: jattn_qkv_weights, rope, q, k, v, B: int, H: int, N_txt: int, N_img: int,
                    N_ref: int, d: int, C: int, stream=None, *, check: bool = True) -> int:
    st = load_library().jattn_qkv_fused(_ptr(x), ctypes.byref(weights) if weights is not None else None,
                                        _ptr(rope), _ptr(q), _ptr(k), _ptr(v), B, H, N_txt, N_img, N_ref, d, C,
                                        _stream(stream))
    if check:
        _check("jattn_qkv_fused", st)
    return st


def repair_count(n: int, rho: float) -> int:
    """Tokens repaired per (b, h) for budget rho: ceil(rho * N), at most N."""
    import math
    return min(n, math.ceil(rho * n - 1e-9)) if rho > 0 else 0


def jattn_fp8_repair_select(k, v, k8, v8, k_scale, v_scale, params: jattn_prologue_params, m: int, err, idx,
                            k_sel, v_sel, B: int, H: int, N_txt: int, N_img: int, N_ref: int, d: int,
                            stream=None, *, check: bool = True) -> int:
    st = load_library().jattn_fp8_repair_select(
        _ptr(k), _ptr(v), _ptr(k8), _ptr(v8), _ptr(k_scale), _ptr(v_scale),
        ctypes.byref(params) if params is not None else None, m, _ptr(err), _ptr(idx), _ptr(k_sel), _ptr(v_sel),
        B, H, N_txt, N_img, N_ref, d, _stream(stream))
    if check:
        _check("jattn_fp8_repair_select", st)
    return st


def jattn_fp8_repair_apply(q8, q_scale, k8, v8, k_scale, v_scale, idx, k_sel, v_sel, m: int, o, lse, B: int,
                           H: int, N_txt: int, N_img: int, N_ref: int, d: int, softmax_scale: float, stream=None,
                           *, check: bool = True) -> int:
    st = load_library().jattn_fp8_repair_apply(
        _ptr(q8), _ptr(q_scale), _ptr(k8), _ptr(v8), _ptr(k_scale), _ptr(v_scale), _ptr(idx), _ptr(k_sel),
        _ptr(v_sel), m, _ptr(o), _ptr(lse), B, H, N_txt, N_img, N_ref, d, softmax_scale, _stream(stream))
    if check:
        _check("jattn_fp8_repair_apply", st)
    return st


def sparse_blocks(n: int) -> tuple:
    """(query blocks, key blocks) of a joint sequence of n tokens."""
    return -(-n // JATTN_SPARSE_QBLOCK), -(-n // JATTN_SPARSE_KBLOCK)


def jattn_sparse_select(q, k, qbar, kbar, probs, kv_idx, kv_cnt, B: int, H: int, N_txt: int, N_img: int,
                        N_ref: int, d: int, softmax_scale: float, tau: float, stream=None, *,
                        check: bool = True) -> int:
    st = load_library().jattn_sparse_select(
        _ptr(q), _ptr(k), _ptr(qbar), _ptr(kbar), _ptr(probs), _ptr(kv_idx), _ptr(kv_cnt),
        B, H, N_txt, N_img, N_ref, d, softmax_scale, tau, _stream(stream))
    if check:
        _check("jattn_sparse_select", st)
    return st


def jattn_sparse_select_noalloc(q, k, probs, kv_idx, kv_cnt, B: int, H: int, N_txt: int, N_img: int, N_ref: int,
                                d: int, softmax_scale: float, tau: float, stream=None, *, check: bool = True) -> int:
    """jattn_sparse_select with the pooled-means workspace inside the library
    (a fixed 16 MiB device array), for callers that cannot allocate."""
    st = load_library().jattn_sparse_select_noalloc(
        _ptr(q), _ptr(k), _ptr(probs), _ptr(kv_idx), _ptr(kv_cnt),
        B, H, N_txt, N_img, N_ref, d, softmax_scale, tau, _stream(stream))
    if check:
        _check("jattn_sparse_select_noalloc", st)
    return st


def jattn_fwd_bf16_sparse(q, k, v, o, lse, kv_idx, kv_cnt, B: int, H: int, N_txt: int, N_img: int, N_ref: int,
                          d: int, softmax_scale: float, stream=None, *, check: bool = True) -> int:
    st = load_library().jattn_fwd_bf16_sparse(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(kv_idx), _ptr(kv_cnt),
        B, H, N_txt, N_img, N_ref, d, softmax_scale, _stream(stream))
    if check:
        _check("jattn_fwd_bf16_sparse", st)
    return st


def jattn_last_cuda_error() -> str:
    return load_library().jattn_last_cuda_error().decode()


def jattn_device_status(stream=None) -> int:
    return load_library().jattn_device_status(_stream(stream))


def jattn_selftest_wait_timeout(timeout_ns: int, stream=None, *, check: bool = True) -> int:
    st = load_library().jattn_selftest_wait_timeout(int(timeout_ns), _stream(stream))
    if check:
        _check("jattn_selftest_wait_timeout", st)
    return st
