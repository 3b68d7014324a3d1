"""Loader for the float64 C oracle (``mfa_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py``; never by the product package. It shares no
code with the CUDA library.

Inputs are numpy arrays holding the exact bit patterns the GPU sees: bf16 as
``uint16``, E4M3 as ``uint8``; int32 for lengths and page tables. Results are
float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mfa_oracle.c")
_LIB = os.path.join(_HERE, "libmfa_oracle.so")
_lock = threading.Lock()
_lib = None

BF16, F32, E4M3 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/libmfa_oracle.so`` (gcc, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-shared", "-fPIC",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            lib.mfa_oracle_decode.restype = ctypes.c_int
            lib.mfa_oracle_decode.argtypes = [
                ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, ctypes.c_int,
                ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                P, ctypes.c_double, ctypes.c_double, ctypes.c_double, P, P, ctypes.c_int, P, P]
            lib.mfa_oracle_combine.restype = None
            lib.mfa_oracle_combine.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P, P]
            lib.mfa_oracle_query_proj.restype = None
            lib.mfa_oracle_query_proj.argtypes = [ctypes.c_int] * 4 + [P, P, P, P]
            lib.mfa_oracle_e4m3_to_double.restype = ctypes.c_double
            lib.mfa_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.mfa_oracle_kv_project.restype = None
            lib.mfa_oracle_kv_project.argtypes = [ctypes.c_int] * 3 + [P, P, P, P, P]
            lib.mfa_oracle_bf16_round.restype = ctypes.c_uint16
            lib.mfa_oracle_bf16_round.argtypes = [ctypes.c_double]
            lib.mfa_oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.mfa_oracle_e4m3_encode.argtypes = [ctypes.c_double]
            lib.mfa_oracle_out_proj.restype = None
            lib.mfa_oracle_out_proj.argtypes = [ctypes.c_int] * 3 + [P, P, P]
            lib.mfa_oracle_gqa_decode.restype = ctypes.c_int
            lib.mfa_oracle_gqa_decode.argtypes = [
                ctypes.c_int] * 4 + [P, P, P, ctypes.c_int64, ctypes.c_int64, P, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, P, ctypes.c_double, P, P]
            lib.mfa_oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return _load().mfa_oracle_num_threads()


def e4m3_to_double(code: int) -> float:
    return _load().mfa_oracle_e4m3_to_double(int(code) & 0xFF)


def decode(q_bits, k, v, seq_lens, scale, *, kv_dtype=BF16, page_table=None, page_size=64,
           k_scale=1.0, v_scale=1.0, select=None):
    """MFA decode attention in float64.

    q_bits: uint16 [B, H, D] (bf16 bits).
    k, v: contiguous cache [B, Lmax, D] or, with ``page_table``, paged
      [num_pages, page_size, D]; uint16 (bf16 bits), float32, or uint8 (E4M3).
    seq_lens: int32 [B]. page_table: int32 [B, max_pages] or None.
    select: optional list of (b, h) pairs; then returns out [n, D], lse [n].
    Returns (out, lse): out [B, H, D] float64, lse [B, H] float64.
    """
    lib = _load()
    q_bits = _c(q_bits, np.uint16)
    B, H, D = q_bits.shape
    cache_dt = {BF16: np.uint16, F32: np.float32, E4M3: np.uint8}[kv_dtype]
    k = _c(k, cache_dt)
    v = _c(v, cache_dt)
    assert k.shape == v.shape and k.shape[-1] == D
    seq_lens = _c(seq_lens, np.int32)
    if page_table is not None:
        page_table = _c(page_table, np.int32)
        num_pages, psize, _ = k.shape
        assert psize == page_size
        max_pages = page_table.shape[1]
        bstride, tstride = 0, 0
    else:
        num_pages, max_pages, psize = 0, 0, 0
        bstride, tstride = k.shape[1] * D, D
    if select is not None:
        sel = np.asarray(select, dtype=np.int32).reshape(-1, 2)
        sel_b = np.ascontiguousarray(sel[:, 0])
        sel_h = np.ascontiguousarray(sel[:, 1])
        n = sel.shape[0]
        out = np.zeros((n, D), np.float64)
        lse = np.zeros((n,), np.float64)
    else:
        sel_b = sel_h = None
        n = 0
        out = np.zeros((B, H, D), np.float64)
        lse = np.zeros((B, H), np.float64)
    rc = lib.mfa_oracle_decode(B, H, D, _ptr(q_bits), _ptr(k), _ptr(v), kv_dtype, bstride, tstride,
                               _ptr(page_table), max_pages, psize, num_pages, _ptr(seq_lens),
                               float(scale), float(k_scale), float(v_scale), _ptr(sel_b),
                               _ptr(sel_h), n, _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle: out-of-range page id or bad argument")
    return out, lse


def gqa_decode(q_bits, k, v, seq_lens, scale, *, page_table=None, page_size=64):
    """Grouped-query decode attention in float64 (bf16 inputs).

    q_bits: uint16 [B, H, D]. k, v: uint16 contiguous [B, Lmax, G, D] or, with
    ``page_table``, paged [num_pages, page_size, G, D]. Head h uses group
    h // (H // G). Returns (out [B, H, D], lse [B, H]) float64.
    """
    lib = _load()
    q_bits = _c(q_bits, np.uint16)
    B, H, D = q_bits.shape
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    assert k.shape == v.shape and k.shape[-1] == D and k.ndim == 4
    G = k.shape[2]
    seq_lens = _c(seq_lens, np.int32)
    if page_table is not None:
        page_table = _c(page_table, np.int32)
        num_pages, psize = k.shape[0], k.shape[1]
        assert psize == page_size
        max_pages = page_table.shape[1]
        bstride, tstride = 0, 0
    else:
        num_pages, max_pages, psize = 0, 0, 0
        bstride, tstride = k.shape[1] * G * D, G * D
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    rc = lib.mfa_oracle_gqa_decode(B, H, G, D, _ptr(q_bits), _ptr(k), _ptr(v), bstride, tstride,
                                   _ptr(page_table), max_pages, psize, num_pages,
                                   _ptr(seq_lens), float(scale), _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle: out-of-range page id or bad argument")
    return out, lse


def combine(parts, part_lse):
    """Merge split partials: parts [n, D] (each normalised over its range), part_lse [n]."""
    lib = _load()
    parts = _c(parts, np.float64)
    part_lse = _c(part_lse, np.float64)
    n, D = parts.shape
    out = np.zeros((D,), np.float64)
    lse = np.zeros((1,), np.float64)
    lib.mfa_oracle_combine(n, D, _ptr(parts), _ptr(part_lse), _ptr(out), _ptr(lse))
    return out, float(lse[0])


def query_proj(x_bits, wqa_bits, wqb_bits):
    """q = (x @ W_qa) @ W_qb in float64 from bf16 bits; x [B, Dm], W_qa [Dm, R], W_qb [R, N]."""
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    wqa_bits = _c(wqa_bits, np.uint16)
    wqb_bits = _c(wqb_bits, np.uint16)
    B, Dm = x_bits.shape
    Dm2, R = wqa_bits.shape
    R2, N = wqb_bits.shape
    assert Dm == Dm2 and R == R2
    out = np.zeros((B, N), np.float64)
    lib.mfa_oracle_query_proj(B, Dm, R, N, _ptr(x_bits), _ptr(wqa_bits), _ptr(wqb_bits), _ptr(out))
    return out


def bf16_round(v: float) -> int:
    """Bits of the bf16 nearest to v (ties to even)."""
    return int(_load().mfa_oracle_bf16_round(float(v)))


def e4m3_encode(v: float) -> int:
    """The E4M3 code nearest to v (ties to an even mantissa, saturating to +-448)."""
    return int(_load().mfa_oracle_e4m3_encode(float(v)))


def kv_project(x_bits, wk_bits, wv_bits):
    """k = x @ W_k, v = x @ W_v in float64 from bf16 bits; x [B, Dm], W [Dm, D]."""
    lib = _load()
    x_bits = _c(x_bits, np.uint16)
    wk_bits = _c(wk_bits, np.uint16)
    wv_bits = _c(wv_bits, np.uint16)
    B, Dm = x_bits.shape
    assert wk_bits.shape == wv_bits.shape and wk_bits.shape[0] == Dm
    D = wk_bits.shape[1]
    k = np.zeros((B, D), np.float64)
    v = np.zeros((B, D), np.float64)
    lib.mfa_oracle_kv_project(B, Dm, D, _ptr(x_bits), _ptr(wk_bits), _ptr(wv_bits), _ptr(k), _ptr(v))
    return k, v


def kv_append(x_bits, wk_bits, wv_bits, k_cache, v_cache, positions, *, kv_dtype=BF16,
              page_table=None, page_size=64, k_scale=1.0, v_scale=1.0):
    """The caches after appending each sequence's new token at row positions[b].

    k_cache, v_cache: contiguous [B, Lmax, D] or paged [num_pages, page_size, D],
    uint16 (bf16 bits) or uint8 (E4M3 codes); page_table int32 [B, max_pages].
    A bf16 cache stores the nearest bf16 of the projected value, an FP8 cache the
    E4M3 code nearest to value / scale. Returns (k_new, v_new, k, v): updated
    copies of the caches and the projected rows in float64.
    """
    k, v = kv_project(x_bits, wk_bits, wv_bits)
    k_new = np.array(k_cache, copy=True)
    v_new = np.array(v_cache, copy=True)
    B, D = k.shape
    for b in range(B):
        t = int(positions[b])
        if page_table is not None:
            page = int(page_table[b][t // page_size])
            if page < 0 or page >= k_new.shape[0]:
                raise ValueError("oracle: out-of-range page id")
            rows = (k_new[page, t % page_size], v_new[page, t % page_size])
        else:
            if t < 0 or t >= k_new.shape[1]:
                raise ValueError("oracle: position outside the cache")
            rows = (k_new[b, t], v_new[b, t])
        for dst, val, scale in ((rows[0], k[b], k_scale), (rows[1], v[b], v_scale)):
            for i in range(D):
                dst[i] = (e4m3_encode(val[i] / scale) if kv_dtype == E4M3
                          else bf16_round(val[i]))
    return k_new, v_new, k, v


def out_proj(o_bits, wo_bits):
    """y = o @ W_o in float64 from bf16 bits; o [B, K] (heads x dim), W_o [K, N]."""
    lib = _load()
    o_bits = _c(o_bits, np.uint16)
    wo_bits = _c(wo_bits, np.uint16)
    B, K = o_bits.shape
    assert wo_bits.shape[0] == K
    N = wo_bits.shape[1]
    y = np.zeros((B, N), np.float64)
    lib.mfa_oracle_out_proj(B, K, N, _ptr(o_bits), _ptr(wo_bits), _ptr(y))
    return y
