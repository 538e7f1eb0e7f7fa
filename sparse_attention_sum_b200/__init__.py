"""Python binding of libdsa, the B200 DSA-layer library (C ABI in include/dsa.h).

Argument marshalling only: every function takes torch CUDA tensors, fills a
``dsa_dims`` struct and calls the entry point of the same name in
``libdsa.so``.  All computation runs in the library's CUDA kernels; there is no
other implementation behind these names.  If ``libdsa.so`` is missing or fails
to load, every call raises :class:`DsaLibraryError` (build it with
``python -m sparse_attention_sum_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

__all__ = [
    "DsaError", "DsaLibraryError", "Dims", "lib", "lib_path", "INVALID", "F32", "BF16",
    "index_scores", "index_scores_fp8", "fp8_quantize", "index_topk", "index_topk_fp8", "topk", "topk_set", "sparse_attend", "layer_forward", "layer_forward_static", "pool_states",
    "expand_selection", "absorb_q", "absorb_out", "index_rotate", "workspace_size", "get_device_status",
    "selftest_wait_timeout", "set_kernel_policy", "last_kernels", "OP_TOPK", "OP_LAYER_FORWARD", "STATUS",
]

INVALID = -1
F32, BF16 = 0, 1
OP_TOPK, OP_LAYER_FORWARD = 1, 2
STATUS = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARGUMENT", 2: "DSA_ERR_UNSUPPORTED",
          3: "DSA_ERR_WORKSPACE", 4: "DSA_ERR_CUDA", 5: "DSA_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.path.join(_HERE, "libdsa.so")


class DsaLibraryError(RuntimeError):
    """libdsa.so could not be loaded: the CUDA path is unavailable."""


class DsaError(RuntimeError):
    def __init__(self, status: int, fn: str, msg: str):
        super().__init__(f"{fn}: {STATUS.get(status, status)}: {msg}")
        self.status = status
        self.name = STATUS.get(status, str(status))


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "batch", "n_q", "n_kv", "idx_heads", "idx_dim", "top_k", "heads", "kv_heads",
        "kd", "vd", "kpool", "out_width", "dtype")]

    def __init__(self, **kw):
        super().__init__()
        for k, v in kw.items():
            setattr(self, k, int(v))

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_}


_VP, _I32P, _F32P = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
_SIGS = {
    "dsa_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "dsa_last_error": ([], ctypes.c_char_p),
    "dsa_version": ([], ctypes.c_char_p),
    "dsa_last_kernels": ([], ctypes.c_char_p),
    "dsa_set_kernel_policy": ([ctypes.c_int], ctypes.c_int),
    "dsa_workspace_size": ([ctypes.POINTER(Dims), ctypes.c_int], ctypes.c_size_t),
    "dsa_index_scores": ([ctypes.POINTER(Dims), _VP, _VP, _F32P, ctypes.c_float, _I32P, _I32P,
                          _I32P, _F32P, _VP], ctypes.c_int),
    "dsa_fp8_quantize": ([ctypes.c_int64, ctypes.c_int32, ctypes.c_int, _VP, ctypes.c_int64, _VP, _F32P, _VP],
                         ctypes.c_int),
    "dsa_index_scores_fp8": ([ctypes.POINTER(Dims), _VP, _F32P, _VP, _F32P, _F32P, ctypes.c_float, _I32P, _I32P,
                              _I32P, _F32P, _VP], ctypes.c_int),
    "dsa_index_topk": ([ctypes.POINTER(Dims), _VP, _VP, _F32P, ctypes.c_float, _I32P, _I32P, _I32P, ctypes.c_int32,
                        _I32P, _VP], ctypes.c_int),
    "dsa_index_topk_fp8": ([ctypes.POINTER(Dims), _VP, _F32P, _VP, _F32P, _F32P, ctypes.c_float, _I32P, _I32P,
                            _I32P, ctypes.c_int32, _I32P, _VP], ctypes.c_int),
    "dsa_topk": ([ctypes.POINTER(Dims), _F32P, _I32P, _I32P, _I32P, ctypes.c_int32, _I32P, _F32P,
                  _VP, ctypes.c_size_t, _VP], ctypes.c_int),
    "dsa_topk_set": ([ctypes.POINTER(Dims), _F32P, _I32P, _I32P, _I32P, ctypes.c_int32, _I32P, _F32P, _VP],
                     ctypes.c_int),
    "dsa_sparse_attend": ([ctypes.POINTER(Dims), _VP, _VP, ctypes.c_int64, _VP, ctypes.c_int64,
                           _I32P, ctypes.c_int32, ctypes.c_float, _VP, _F32P, _VP], ctypes.c_int),
    "dsa_layer_forward": ([ctypes.POINTER(Dims), _VP, _VP, _F32P, ctypes.c_float, _I32P, _I32P,
                           _I32P, _VP, _VP, ctypes.c_int64, _VP, ctypes.c_int64, ctypes.c_float,
                           _I32P, _I32P, _VP, _F32P, _VP, ctypes.c_size_t, _VP], ctypes.c_int),
    "dsa_layer_forward_static": ([ctypes.POINTER(Dims), _VP, _VP, _F32P, ctypes.c_float, _I32P, _I32P,
                                  _I32P, _VP, _VP, ctypes.c_int64, _VP, ctypes.c_int64, ctypes.c_float,
                                  _I32P, _I32P, _VP, _F32P, _VP], ctypes.c_int),
    "dsa_pool_states": ([ctypes.POINTER(Dims), _VP, _VP, _F32P, _F32P, ctypes.c_float, _I32P,
                         _I32P, _VP, _I32P, _VP], ctypes.c_int),
    "dsa_expand_selection": ([ctypes.POINTER(Dims), _I32P, _I32P, _I32P, _I32P, _I32P, _I32P,
                              _VP], ctypes.c_int),
    "dsa_absorb_q": ([ctypes.POINTER(Dims), _VP, ctypes.c_int32, _VP, ctypes.c_int32, _VP, _VP],
                     ctypes.c_int),
    "dsa_absorb_out": ([ctypes.POINTER(Dims), _VP, ctypes.c_int32, _VP, ctypes.c_int32, _VP, _VP],
                       ctypes.c_int),
    "dsa_index_rotate": ([ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                          ctypes.c_int32, _F32P, _F32P, ctypes.c_float, ctypes.c_int32, _I32P, ctypes.c_int,
                          _VP, ctypes.c_int64, ctypes.c_int, _VP, ctypes.c_int64, _I32P, ctypes.c_int64, _VP],
                         ctypes.c_int),
    "dsa_get_device_status": ([_VP], ctypes.c_int),
    "dsa_selftest_wait_timeout": ([ctypes.c_int64, _VP], ctypes.c_int),
}

_lib = None


def lib():
    """The loaded ``libdsa.so`` (ctypes.CDLL); raises DsaLibraryError if unavailable."""
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            raise DsaLibraryError(f"{path} not found: build it with python -m sparse_attention_sum_b200.build")
        try:
            h = ctypes.CDLL(path, mode=ctypes.RTLD_GLOBAL)
        except OSError as e:
            raise DsaLibraryError(f"cannot load {path}: {e}") from e
        for name, (args, res) in _SIGS.items():
            fn = getattr(h, name)
            fn.argtypes = args
            fn.restype = res
        _lib = h
    return _lib


def _ptr(t, dense: bool = True) -> Optional[int]:
    """Device address of tensor ``t``.  The C ABI reads dense row-major arrays except where a row-stride
    argument accompanies the pointer (``dense=False``: only the innermost axis must be contiguous)."""
    if t is None:
        return None
    if dense and not t.is_contiguous():
        raise ValueError("libdsa entry points take contiguous tensors (row-major, no gaps) for this argument")
    if not dense and t.dim() > 0 and t.stride(-1) != 1:
        raise ValueError("the innermost axis of a strided argument must be contiguous")
    if not t.is_cuda:
        raise ValueError("libdsa entry points take CUDA tensors")
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(status: int, fn: str):
    if status != 0:
        raise DsaError(status, fn, lib().dsa_last_error().decode())


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def last_kernels() -> list:
    """Kernel families the most recent libdsa call on this thread launched, in order."""
    s = lib().dsa_last_kernels().decode()
    return s.split(",") if s else []


def set_kernel_policy(policy: int) -> int:
    return lib().dsa_set_kernel_policy(int(policy))


def workspace_size(dims: Dims, op: int) -> int:
    return int(lib().dsa_workspace_size(ctypes.byref(dims), op))


def index_scores(dims: Dims, q_idx, k_idx, w, scale: float, q_pos, kv_start, kv_len, scores,
                 stream=None):
    _check(lib().dsa_index_scores(ctypes.byref(dims), _ptr(q_idx), _ptr(k_idx), _ptr(w), scale,
                                  _ptr(q_pos), _ptr(kv_start), _ptr(kv_len), _ptr(scores),
                                  _stream(stream)), "dsa_index_scores")


def fp8_quantize(x, codes, scales, stream=None):
    """dsa_fp8_quantize: per-vector e4m3 codes and fp32 scales of ``x [..., 128]`` (bf16 or fp32; rows may
    be strided).  ``codes`` is a uint8 tensor ``[..., 128]``, ``scales`` fp32 ``[...]``."""
    if x.shape[-1] != 128 or x.stride(-1) != 1:
        raise ValueError("x must end in a contiguous axis of 128 values")
    rows = x.reshape(-1, 128) if x.is_contiguous() else x.view(-1, 128)
    if codes.dtype != __import__("torch").uint8 or codes.numel() != rows.shape[0] * 128:
        raise ValueError("codes must be a uint8 tensor of x's shape")
    if scales.numel() != rows.shape[0]:
        raise ValueError("scales must hold one value per row of x")
    _check(lib().dsa_fp8_quantize(int(rows.shape[0]), 128, _dtype_code(x), _ptr(rows, False), int(rows.stride(0)),
                                  _ptr(codes), _ptr(scales), _stream(stream)), "dsa_fp8_quantize")


def index_scores_fp8(dims: Dims, q_codes, q_scales, k_codes, k_scales, w, scale: float, q_pos, kv_start, kv_len,
                     scores, stream=None):
    _check(lib().dsa_index_scores_fp8(ctypes.byref(dims), _ptr(q_codes), _ptr(q_scales), _ptr(k_codes),
                                      _ptr(k_scales), _ptr(w), scale, _ptr(q_pos), _ptr(kv_start), _ptr(kv_len),
                                      _ptr(scores), _stream(stream)), "dsa_index_scores_fp8")


def index_topk(dims: Dims, q_idx, k_idx, w, scale: float, q_pos, kv_start, kv_len, k: int, idx, stream=None):
    """dsa_index_topk: the selection (ascending key order) straight from the indexer inputs."""
    _check(lib().dsa_index_topk(ctypes.byref(dims), _ptr(q_idx), _ptr(k_idx), _ptr(w), scale, _ptr(q_pos),
                                _ptr(kv_start), _ptr(kv_len), int(k), _ptr(idx), _stream(stream)), "dsa_index_topk")


def index_topk_fp8(dims: Dims, q_codes, q_scales, k_codes, k_scales, w, scale: float, q_pos, kv_start, kv_len,
                   k: int, idx, stream=None):
    """dsa_index_topk_fp8: the FP8 selection (ascending key order) straight from the e4m3 operands."""
    _check(lib().dsa_index_topk_fp8(ctypes.byref(dims), _ptr(q_codes), _ptr(q_scales), _ptr(k_codes),
                                    _ptr(k_scales), _ptr(w), scale, _ptr(q_pos), _ptr(kv_start), _ptr(kv_len), int(k),
                                    _ptr(idx), _stream(stream)), "dsa_index_topk_fp8")


def topk(dims: Dims, scores, q_pos, kv_start, kv_len, k: int, idx, vals=None, ws=None,
         stream=None):
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().dsa_topk(ctypes.byref(dims), _ptr(scores), _ptr(q_pos), _ptr(kv_start),
                          _ptr(kv_len), int(k), _ptr(idx), _ptr(vals), _ptr(ws), wsb,
                          _stream(stream)), "dsa_topk")


def topk_set(dims: Dims, scores, q_pos, kv_start, kv_len, k: int, idx, vals=None, stream=None):
    """dsa_topk's selection listed in ascending key order (the fused layer's form)."""
    _check(lib().dsa_topk_set(ctypes.byref(dims), _ptr(scores), _ptr(q_pos), _ptr(kv_start), _ptr(kv_len),
                              int(k), _ptr(idx), _ptr(vals), _stream(stream)), "dsa_topk_set")


def sparse_attend(dims: Dims, q, k, k_row_stride: int, v, v_row_stride: int, idx, width: int,
                  scale: float, out, lse=None, stream=None):
    _check(lib().dsa_sparse_attend(ctypes.byref(dims), _ptr(q), _ptr(k, False), int(k_row_stride), _ptr(v, False),
                                   int(v_row_stride), _ptr(idx), int(width), scale, _ptr(out),
                                   _ptr(lse), _stream(stream)), "dsa_sparse_attend")


def layer_forward(dims: Dims, q_idx, k_idx, w, idx_scale: float, q_pos, kv_start, kv_len, q, k,
                  k_row_stride: int, v, v_row_stride: int, attn_scale: float, out, lse=None,
                  idx_in=None, idx_out=None, ws=None, stream=None):
    wsb = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib().dsa_layer_forward(ctypes.byref(dims), _ptr(q_idx), _ptr(k_idx), _ptr(w), idx_scale,
                                   _ptr(q_pos), _ptr(kv_start), _ptr(kv_len), _ptr(q), _ptr(k, False),
                                   int(k_row_stride), _ptr(v, False), int(v_row_stride), attn_scale,
                                   _ptr(idx_in), _ptr(idx_out), _ptr(out), _ptr(lse), _ptr(ws), wsb,
                                   _stream(stream)), "dsa_layer_forward")


def layer_forward_static(dims: Dims, q_idx, k_idx, w, idx_scale: float, q_pos, kv_start, kv_len, q, k,
                         k_row_stride: int, v, v_row_stride: int, attn_scale: float, out, lse=None,
                         idx_in=None, idx_out=None, stream=None):
    """dsa_layer_forward with the library's fixed scratch array (no workspace argument)."""
    _check(lib().dsa_layer_forward_static(ctypes.byref(dims), _ptr(q_idx), _ptr(k_idx), _ptr(w), idx_scale,
                                          _ptr(q_pos), _ptr(kv_start), _ptr(kv_len), _ptr(q), _ptr(k, False),
                                          int(k_row_stride), _ptr(v, False), int(v_row_stride), attn_scale,
                                          _ptr(idx_in), _ptr(idx_out), _ptr(out), _ptr(lse), _stream(stream)),
           "dsa_layer_forward_static")


def pool_states(dims: Dims, k, gate, ln_w, ln_b, ln_eps: float, kv_start, kv_len, pooled, n_pools,
                stream=None):
    _check(lib().dsa_pool_states(ctypes.byref(dims), _ptr(k), _ptr(gate), _ptr(ln_w), _ptr(ln_b),
                                 ln_eps, _ptr(kv_start), _ptr(kv_len), _ptr(pooled), _ptr(n_pools),
                                 _stream(stream)), "dsa_pool_states")


def expand_selection(dims: Dims, pool_idx, q_pos, kv_start, kv_len, n_pools, tok_idx, stream=None):
    _check(lib().dsa_expand_selection(ctypes.byref(dims), _ptr(pool_idx), _ptr(q_pos), _ptr(kv_start),
                                      _ptr(kv_len), _ptr(n_pools), _ptr(tok_idx), _stream(stream)),
           "dsa_expand_selection")


def absorb_q(dims: Dims, q, d: int, w_uk, L: int, q_lat, stream=None):
    _check(lib().dsa_absorb_q(ctypes.byref(dims), _ptr(q), int(d), _ptr(w_uk), int(L), _ptr(q_lat),
                              _stream(stream)), "dsa_absorb_q")


def absorb_out(dims: Dims, o_lat, L: int, w_uv, e: int, out, stream=None):
    _check(lib().dsa_absorb_out(ctypes.byref(dims), _ptr(o_lat), int(L), _ptr(w_uv), int(e), _ptr(out),
                                _stream(stream)), "dsa_absorb_out")


def index_rotate(x, out, n_rope: int, rope_theta: float, pos=None, layer_norm: bool = False, ln_w=None,
                 ln_b=None, ln_eps: float = 0.0, hadamard: bool = True, out_rows=None, stream=None):
    """dsa_index_rotate: prepare indexer queries or keys.

    ``x`` is ``[n_rows, heads, dim]`` and ``out`` is ``[capacity, heads, dim]``, each with its
    last two axes contiguous (the row stride may be larger).  Row r goes to ``out[out_rows[r]]``
    (or ``out[r]``)."""
    for name, t in (("x", x), ("out", out)):
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must be [rows, heads, dim] with contiguous heads and values")
    if out.shape[1:] != x.shape[1:]:
        raise ValueError("x and out must have the same heads and dim")
    n_rows, heads, dim = x.shape
    _check(lib().dsa_index_rotate(int(n_rows), int(heads), int(dim), int(n_rope), float(rope_theta),
                                  int(bool(layer_norm)), _ptr(ln_w), _ptr(ln_b), float(ln_eps), int(bool(hadamard)),
                                  _ptr(pos), _dtype_code(x), _ptr(x, False), int(x.stride(0)), _dtype_code(out),
                                  _ptr(out, False), int(out.stride(0)), _ptr(out_rows), int(out.shape[0]),
                                  _stream(stream)),
           "dsa_index_rotate")


def get_device_status(stream=None) -> int:
    """Synchronize and return (and clear) the device status code (0 = DSA_OK)."""
    return int(lib().dsa_get_device_status(_stream(stream)))


def selftest_wait_timeout(timeout_ns: int, stream=None):
    _check(lib().dsa_selftest_wait_timeout(int(timeout_ns), _stream(stream)), "dsa_selftest_wait_timeout")
