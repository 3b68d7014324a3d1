"""Python binding of libmfa.so (C ABI in ``include/mfa.h``).

Argument marshalling only: torch tensors become ``mfa_tensor`` descriptors,
the current CUDA stream is passed through, and every step of the computation
runs in the library's kernels. There is no fallback: if ``libmfa.so`` is
missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmfa.so")

MFA_BF16, MFA_F32, MFA_FP8_E4M3, MFA_I32 = 0, 1, 2, 3
STATUS = {
    0: "MFA_OK", 1: "MFA_ERR_INVALID_ARG", 2: "MFA_ERR_UNSUPPORTED", 3: "MFA_ERR_CUDA",
    4: "MFA_ERR_WORKSPACE", 5: "MFA_ERR_BAD_INDEX", 6: "MFA_ERR_TIMEOUT",
}
STATUS_CODES = {v: k for k, v in STATUS.items()}
H, D = 64, 256


class MfaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS.get(code, code)}")
        self.code = code


class MfaTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


_lib = None
_lock = threading.Lock()

EXPORTS = ("mfa_decode_attention", "mfa_decode_attention_ex", "mfa_decode_workspace_size",
           "mfa_query_proj", "mfa_query_proj_ex", "mfa_query_proj_workspace_size",
           "mfa_kv_append", "mfa_kv_append_workspace_size",
           "mfa_output_proj", "mfa_output_proj_workspace_size", "mfa_lse_merge",
           "mfa_read_status", "mfa_error_string", "mfa_version", "mfa_last_cuda_error_string",
           "mfa_decode_attention_noalloc", "mfa_selftest_wait_timeout",
           "mfa_gqa_decode_attention", "mfa_qproj_decode_attention",
           "mfa_qproj_decode_workspace_size")


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m decode_attention_08_b200.build`"
                    " (there is no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            P, T = ctypes.c_void_p, ctypes.POINTER(MfaTensor)
            L.mfa_decode_attention.argtypes = [T, T, T, T, T, T, ctypes.c_float, ctypes.c_int, P]
            L.mfa_decode_attention.restype = ctypes.c_int
            L.mfa_decode_attention_ex.argtypes = [T, T, T, T, T, T, ctypes.c_float, ctypes.c_int,
                                                  ctypes.c_float, ctypes.c_float, ctypes.c_int, T,
                                                  P, ctypes.c_size_t, P]
            L.mfa_decode_attention_ex.restype = ctypes.c_int
            L.mfa_decode_attention_noalloc.argtypes = [T, T, T, T, T, T, ctypes.c_float,
                                                       ctypes.c_int, ctypes.c_float,
                                                       ctypes.c_float, ctypes.c_int, T, P]
            L.mfa_decode_attention_noalloc.restype = ctypes.c_int
            L.mfa_decode_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int]
            L.mfa_decode_workspace_size.restype = ctypes.c_size_t
            L.mfa_query_proj.argtypes = [T, T, T, T, P]
            L.mfa_query_proj.restype = ctypes.c_int
            L.mfa_query_proj_ex.argtypes = [T, T, T, T, P, ctypes.c_size_t, P]
            L.mfa_query_proj_ex.restype = ctypes.c_int
            L.mfa_query_proj_workspace_size.argtypes = [ctypes.c_int] * 3
            L.mfa_query_proj_workspace_size.restype = ctypes.c_size_t
            L.mfa_kv_append.argtypes = [T, T, T, T, T, T, T, ctypes.c_int, ctypes.c_float,
                                        ctypes.c_float, P, ctypes.c_size_t, P]
            L.mfa_kv_append.restype = ctypes.c_int
            L.mfa_kv_append_workspace_size.argtypes = [ctypes.c_int, ctypes.c_int]
            L.mfa_kv_append_workspace_size.restype = ctypes.c_size_t
            L.mfa_output_proj.argtypes = [T, T, T, P, ctypes.c_size_t, P]
            L.mfa_output_proj.restype = ctypes.c_int
            L.mfa_output_proj_workspace_size.argtypes = [ctypes.c_int] * 3
            L.mfa_output_proj_workspace_size.restype = ctypes.c_size_t
            L.mfa_lse_merge.argtypes = [T, T, T, T, P]
            L.mfa_lse_merge.restype = ctypes.c_int
            L.mfa_gqa_decode_attention.argtypes = [T, T, T, T, T, T, ctypes.c_float, ctypes.c_int,
                                                   T, P, ctypes.c_size_t, P]
            L.mfa_gqa_decode_attention.restype = ctypes.c_int
            L.mfa_qproj_decode_attention.argtypes = [T, T, T, T, T, T, T, T, T, ctypes.c_float,
                                                     ctypes.c_int, ctypes.c_float, ctypes.c_float,
                                                     ctypes.c_int, T, P, ctypes.c_size_t, P]
            L.mfa_qproj_decode_attention.restype = ctypes.c_int
            L.mfa_qproj_decode_workspace_size.argtypes = [ctypes.c_int] * 4
            L.mfa_qproj_decode_workspace_size.restype = ctypes.c_size_t
            L.mfa_selftest_wait_timeout.argtypes = [ctypes.c_ulonglong, P]
            L.mfa_selftest_wait_timeout.restype = ctypes.c_int
            L.mfa_read_status.argtypes = [P, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
            L.mfa_read_status.restype = ctypes.c_int
            L.mfa_error_string.argtypes = [ctypes.c_int]
            L.mfa_error_string.restype = ctypes.c_char_p
            L.mfa_last_cuda_error_string.argtypes = []
            L.mfa_last_cuda_error_string.restype = ctypes.c_char_p
            L.mfa_version.argtypes = []
            L.mfa_version.restype = ctypes.c_int
            _lib = L
    return _lib


_DTYPES = {torch.bfloat16: MFA_BF16, torch.float32: MFA_F32, torch.uint8: MFA_FP8_E4M3,
           torch.float8_e4m3fn: MFA_FP8_E4M3, torch.int32: MFA_I32}


def describe(t: Optional[torch.Tensor]):
    """ctypes pointer to an mfa_tensor describing ``t`` (None -> NULL)."""
    if t is None:
        return None
    if t.dtype not in _DTYPES:
        raise TypeError(f"unsupported dtype {t.dtype}")
    d = MfaTensor()
    d.data = t.data_ptr()
    d.dtype = _DTYPES[t.dtype]
    d.ndim = t.dim()
    for i in range(t.dim()):
        d.shape[i] = t.shape[i]
        d.stride[i] = t.stride(i)
    return ctypes.pointer(d)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(rc: int, what: str):
    if rc == 3:
        raise MfaError(rc, f"{what} ({lib().mfa_last_cuda_error_string().decode()})")
    if rc != 0:
        raise MfaError(rc, what)


def _kv_code(kv_dtype) -> int:
    if kv_dtype in ("bf16", MFA_BF16, torch.bfloat16):
        return MFA_BF16
    if kv_dtype in ("e4m3", "fp8", MFA_FP8_E4M3, torch.float8_e4m3fn, torch.uint8):
        return MFA_FP8_E4M3
    raise ValueError(f"kv_dtype {kv_dtype!r}")


def decode_attention(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale=1.0 / 16,
                     kv_dtype="bf16", stream=None):
    """``mfa_decode_attention``: out = softmax(scale q K^T) V per head over each sequence."""
    rc = lib().mfa_decode_attention(describe(q), describe(k_cache), describe(v_cache),
                                    describe(page_table), describe(seq_lens), describe(out),
                                    float(softmax_scale), _kv_code(kv_dtype), _stream(stream))
    _check(rc, "mfa_decode_attention")
    return out


def decode_workspace_size(batch: int, num_splits: int = 0) -> int:
    return int(lib().mfa_decode_workspace_size(int(batch), int(num_splits)))


def decode_attention_ex(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale=1.0 / 16,
                        kv_dtype="bf16", k_scale=1.0, v_scale=1.0, num_splits=0, lse_out=None,
                        workspace: Optional[torch.Tensor] = None, stream=None):
    """``mfa_decode_attention_ex`` (scales, split control, lse, caller workspace)."""
    need = decode_workspace_size(q.shape[0], num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)  # needs no zeroing
    rc = lib().mfa_decode_attention_ex(
        describe(q), describe(k_cache), describe(v_cache), describe(page_table),
        describe(seq_lens), describe(out), float(softmax_scale), _kv_code(kv_dtype),
        float(k_scale), float(v_scale), int(num_splits), describe(lse_out),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mfa_decode_attention_ex")
    return out


def decode_attention_noalloc(q, k_cache, v_cache, page_table, seq_lens, out,
                             softmax_scale=1.0 / 16, kv_dtype="bf16", k_scale=1.0, v_scale=1.0,
                             num_splits=0, lse_out=None, stream=None):
    """``mfa_decode_attention_noalloc``: as ``decode_attention_ex`` but the split
    workspace is the library's fixed device array, so no device memory is
    allocated for the call (for callers that cannot allocate). Calls that
    overlap on the GPU share that array and must be serialised."""
    rc = lib().mfa_decode_attention_noalloc(
        describe(q), describe(k_cache), describe(v_cache), describe(page_table),
        describe(seq_lens), describe(out), float(softmax_scale), _kv_code(kv_dtype),
        float(k_scale), float(v_scale), int(num_splits), describe(lse_out), _stream(stream))
    _check(rc, "mfa_decode_attention_noalloc")
    return out


def gqa_decode_attention(q, k_cache, v_cache, page_table, seq_lens, out,
                         softmax_scale=1.0 / 128 ** 0.5, num_splits=0, lse_out=None,
                         workspace: Optional[torch.Tensor] = None, stream=None):
    """``mfa_gqa_decode_attention``: grouped-query decode attention, q [B, 64, 128],
    caches [.., 2, 128] bf16 (heads 0-31 use group 0, 32-63 group 1)."""
    need = decode_workspace_size(q.shape[0], num_splits)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    rc = lib().mfa_gqa_decode_attention(
        describe(q), describe(k_cache), describe(v_cache), describe(page_table),
        describe(seq_lens), describe(out), float(softmax_scale), int(num_splits),
        describe(lse_out), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(rc, "mfa_gqa_decode_attention")
    return out


def qproj_decode_workspace_size(batch: int, dm: int, rank: int, num_splits: int = 0) -> int:
    return int(lib().mfa_qproj_decode_workspace_size(int(batch), int(dm), int(rank),
                                                     int(num_splits)))


def qproj_decode_attention(x, w_qa, w_qb, q_out, k_cache, v_cache, page_table, seq_lens, out,
                           softmax_scale=1.0 / 16, kv_dtype="bf16", k_scale=1.0, v_scale=1.0,
                           num_splits=0, lse_out=None, workspace: Optional[torch.Tensor] = None,
                           stream=None):
    """``mfa_qproj_decode_attention``: q_out = (x W_qa) W_qb, then decode attention
    of q_out (as [B, 64, 256]) over the caches, in one call. A workspace passed
    in must have had its first 4 KB zeroed before its first use."""
    if workspace is None:
        workspace = torch.zeros(qproj_decode_workspace_size(x.shape[0], x.shape[1],
                                                            w_qa.shape[1], num_splits),
                                dtype=torch.uint8, device=x.device)
    rc = lib().mfa_qproj_decode_attention(
        describe(x), describe(w_qa), describe(w_qb), describe(q_out), describe(k_cache),
        describe(v_cache), describe(page_table), describe(seq_lens), describe(out),
        float(softmax_scale), _kv_code(kv_dtype), float(k_scale), float(v_scale),
        int(num_splits), describe(lse_out), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mfa_qproj_decode_attention")
    return out


def query_proj(x, w_qa, w_qb, q_out, stream=None):
    """``mfa_query_proj``: q_out = (x W_qa) W_qb."""
    rc = lib().mfa_query_proj(describe(x), describe(w_qa), describe(w_qb), describe(q_out),
                              _stream(stream))
    _check(rc, "mfa_query_proj")
    return q_out


def query_proj_workspace_size(batch: int, dm: int, rank: int) -> int:
    return int(lib().mfa_query_proj_workspace_size(int(batch), int(dm), int(rank)))


def query_proj_ex(x, w_qa, w_qb, q_out, workspace: torch.Tensor, stream=None):
    rc = lib().mfa_query_proj_ex(describe(x), describe(w_qa), describe(w_qb), describe(q_out),
                                 workspace.data_ptr(),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mfa_query_proj_ex")
    return q_out


def kv_append_workspace_size(batch: int, hidden: int) -> int:
    return int(lib().mfa_kv_append_workspace_size(int(batch), int(hidden)))


def kv_append(x, w_k, w_v, k_cache, v_cache, positions, page_table=None, kv_dtype="bf16",
              k_scale: float = 1.0, v_scale: float = 1.0, workspace=None, stream=None):
    """``mfa_kv_append``: writes each sequence's new key/value row (x W_k, x W_v)
    into the caches at row ``positions[b]``. ``workspace`` is allocated here when
    not given."""
    if workspace is None:
        n = kv_append_workspace_size(x.shape[0], x.shape[1])
        if n == 0:
            raise RuntimeError("mfa_kv_append_workspace_size failed")
        workspace = torch.empty(n, dtype=torch.uint8, device=x.device)
    rc = lib().mfa_kv_append(describe(x), describe(w_k), describe(w_v), describe(k_cache),
                             describe(v_cache),
                             None if page_table is None else describe(page_table),
                             describe(positions), _kv_code(kv_dtype), float(k_scale),
                             float(v_scale), workspace.data_ptr(),
                             workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mfa_kv_append")
    return k_cache, v_cache


def output_proj_workspace_size(batch: int, k: int, n: int) -> int:
    return int(lib().mfa_output_proj_workspace_size(int(batch), int(k), int(n)))


def output_proj(o, w_o, y, workspace=None, stream=None):
    """``mfa_output_proj``: y = o W_o (o [B, K] = attention outputs, heads x dim)."""
    if workspace is None:
        n = output_proj_workspace_size(o.shape[0], o.shape[1], w_o.shape[1])
        if n == 0:
            raise RuntimeError("mfa_output_proj_workspace_size failed")
        workspace = torch.empty(n, dtype=torch.uint8, device=o.device)
    rc = lib().mfa_output_proj(describe(o), describe(w_o), describe(y), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mfa_output_proj")
    return y


def lse_merge(o_parts, lse_parts, out, lse_out=None, stream=None):
    """``mfa_lse_merge``: merge attention parts over disjoint key ranges
    (o_parts [S, B, 64, 256] f32, lse_parts [S, B, 64] f32) into out [B, 64, 256]."""
    rc = lib().mfa_lse_merge(describe(o_parts), describe(lse_parts), describe(out),
                             describe(lse_out), _stream(stream))
    _check(rc, "mfa_lse_merge")
    return out


def selftest_wait_timeout(wait_ns: int, stream=None) -> None:
    """``mfa_selftest_wait_timeout``: make one bounded in-kernel wait run out
    (no fault); read the resulting MFA_ERR_TIMEOUT with ``read_status``."""
    _check(lib().mfa_selftest_wait_timeout(int(wait_ns), _stream(stream)),
           "mfa_selftest_wait_timeout")


def read_status(stream=None, reset: bool = True) -> int:
    """Synchronise ``stream`` and read the device status word (0 = no error)."""
    v = ctypes.c_int(0)
    _check(lib().mfa_read_status(_stream(stream), int(bool(reset)), ctypes.byref(v)),
           "mfa_read_status")
    return v.value


def error_string(code: int) -> str:
    return lib().mfa_error_string(int(code)).decode()


def version() -> int:
    return int(lib().mfa_version())
