"""NumPy float64 twin of the C oracle: a second, independent restatement of the
same definitions, used only to cross-check ``mfa_oracle.c``.

TEST INFRASTRUCTURE ONLY (see ``oracle.py``). Shares no code with the C oracle or
with the CUDA library.

Definitions (Step-3 page, "Key points -> Architecture": 64 query heads share one
key head and one value head of dimension 256; queries come from a 2048-wide
bottleneck over the 7168-wide hidden state):
  attention   out[b,h] = softmax(scale * q[b,h] @ K_b^T) @ V_b over the first L_b tokens
  projection  q = (x @ W_qa) @ W_qb
Empty sequences give a zero output and lse = -inf.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits):
    """Exact up-conversion: bf16 bits are the high half of a binary32."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def e4m3_to_f64(codes):
    """OCP E4M3 (e4m3fn) codes -> float64, from the format's field definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    mag = np.where(e == 0, sub, normal)
    mag = np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, mag)
    return sign * mag


def _dequant(cache, kv_dtype):
    if kv_dtype == 2:
        return e4m3_to_f64(cache)
    if kv_dtype == 1:
        return np.asarray(cache, dtype=np.float32).astype(np.float64)
    return bf16_bits_to_f64(cache)


def gather_sequence(cache, b, L, page_table=None, page_size=64):
    """Rows [0, L) of sequence b: slab cache[b, :L] or page-table gather."""
    if page_table is None:
        return cache[b, :L]
    t = np.arange(L)
    pages = np.asarray(page_table)[b, t // page_size]
    return cache[pages, t % page_size]


def decode(q_bits, k, v, seq_lens, scale, *, kv_dtype=0, page_table=None, page_size=64,
           k_scale=1.0, v_scale=1.0):
    """Returns out [B, H, D], lse [B, H] (float64)."""
    q = bf16_bits_to_f64(q_bits)
    B, H, D = q.shape
    kd = _dequant(k, kv_dtype) * k_scale
    vd = _dequant(v, kv_dtype) * v_scale
    out = np.zeros((B, H, D), np.float64)
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        if L <= 0:
            continue
        Kb = gather_sequence(kd, b, L, page_table, page_size)
        Vb = gather_sequence(vd, b, L, page_table, page_size)
        s = scale * (q[b] @ Kb.T)                      # [H, L]
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        denom = e.sum(axis=1, keepdims=True)
        out[b] = (e / denom) @ Vb
        lse[b] = (m + np.log(denom))[:, 0]
    return out, lse


def gqa_decode(q_bits, k, v, seq_lens, scale, *, page_table=None, page_size=64):
    """Grouped-query attention: q [B, H, D] bf16 bits, caches [.., G, D] bf16 bits;
    the H heads form G consecutive groups, group g attends over key/value head g.
    Returns out [B, H, D], lse [B, H]."""
    q = bf16_bits_to_f64(q_bits)
    B, H, D = q.shape
    kd, vd = bf16_bits_to_f64(k), bf16_bits_to_f64(v)
    G = kd.shape[-2]
    out = np.zeros((B, H, D), np.float64)
    lse = np.full((B, H), -np.inf)
    for b in range(B):
        L = int(seq_lens[b])
        if L <= 0:
            continue
        Kb = gather_sequence(kd, b, L, page_table, page_size)     # [L, G, D]
        Vb = gather_sequence(vd, b, L, page_table, page_size)
        qg = q[b].reshape(G, H // G, D)                           # [G, H/G, D]
        s = scale * np.einsum("gjd,tgd->gjt", qg, Kb)             # [G, H/G, L]
        m = s.max(axis=2, keepdims=True)
        e = np.exp(s - m)
        denom = e.sum(axis=2, keepdims=True)
        out[b] = np.einsum("gjt,tgd->gjd", e / denom, Vb).reshape(H, D)
        lse[b] = (m + np.log(denom)).reshape(H)
    return out, lse


def combine(parts, part_lse):
    """Flash-Decoding merge of per-range normalised partials."""
    parts = np.asarray(parts, np.float64)
    part_lse = np.asarray(part_lse, np.float64)
    m = part_lse.max()
    if m == -np.inf:
        return np.zeros(parts.shape[1]), -np.inf
    w = np.exp(part_lse - m)
    return (w[:, None] * parts).sum(0) / w.sum(), m + np.log(w.sum())


def query_proj(x_bits, wqa_bits, wqb_bits):
    x = bf16_bits_to_f64(x_bits)
    return (x @ bf16_bits_to_f64(wqa_bits)) @ bf16_bits_to_f64(wqb_bits)


def kv_project(x_bits, wk_bits, wv_bits):
    x = bf16_bits_to_f64(x_bits)
    return x @ bf16_bits_to_f64(wk_bits), x @ bf16_bits_to_f64(wv_bits)


def out_proj(o_bits, wo_bits):
    return bf16_bits_to_f64(o_bits) @ bf16_bits_to_f64(wo_bits)
