"""Seeded synthetic inputs for MFA decode attention and the MFA query projection.

This module only draws and lays out inputs; it holds none of the method's
arithmetic. Both the CUDA path and the float64 oracle consume exactly what it
returns (bf16 tensors, E4M3 codes, int32 lengths and page tables).

Shapes follow the Step-3 page ("Key points -> Architecture"): 64 query heads of
dimension 256 sharing one key head and one value head of dimension 256; hidden
size 7168; query bottleneck 2048. The workloads follow the pages' deployment
setting (4K context, large decode batches, BF16 and FP8 attention); all values
are synthetic (the pages' weights and traffic are not available).

Recipe (every draw from one CPU ``torch.Generator`` seeded with ``seed``):
  * q, K, V ~ N(0, 1) drawn in float32, rounded to bf16 (round-to-nearest-even).
  * FP8 caches: K and V are drawn as above (bf16), then per tensor
    ``scale = amax(|X|) / 448`` (float32) and ``code = e4m3fn(X / scale)``.
  * Paged caches: the pool holds exactly sum_b ceil(L_b / page) pages; logical
    page j of sequence b (enumerated in (b, j) order) is placed at physical page
    perm[idx] for a seeded permutation perm; page-table entries past a sequence's
    last page are -1; rows past L_b inside the last page are NaN (bf16) or the
    E4M3 NaN code, so any over-read shows up.
  * Contiguous caches with L_b < Lmax are NaN-filled past L_b for the same reason.
  * Projection: x ~ N(0, 1), W_qa, W_qb ~ N(0, 0.02^2) (0.02 is the standard
    deviation), all bf16.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

H = 64          # query heads
D = 256         # head dimension (shared K head and V head)
HIDDEN = 7168   # model hidden size
RANK = 2048     # query low-rank bottleneck
E4M3_MAX = 448.0
E4M3_NAN = 0x7F
_CHUNK = 1 << 24


def _randn_bf16(g: torch.Generator, shape, std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) in float32, drawn in fixed-size chunks, rounded to bf16 (RNE)."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.bfloat16)
    for s in range(0, n, _CHUNK):
        e = min(n, s + _CHUNK)
        chunk = torch.randn(e - s, generator=g, dtype=torch.float32)
        if std != 1.0:
            chunk.mul_(std)
        out[s:e] = chunk.to(torch.bfloat16)
    return out.view(*shape)


def quantize_e4m3(x_bf16: torch.Tensor):
    """Per-tensor E4M3 encoding of the drawn cache: (codes uint8, scale float)."""
    amax = x_bf16.abs().max().to(torch.float32).item()
    scale = float(torch.tensor(amax / E4M3_MAX, dtype=torch.float32).item()) if amax > 0 else 1.0
    codes = torch.empty(x_bf16.shape, dtype=torch.uint8)
    flat_in = x_bf16.reshape(-1)
    flat_out = codes.view(-1)
    for s in range(0, flat_in.numel(), _CHUNK):
        e = min(flat_in.numel(), s + _CHUNK)
        q = (flat_in[s:e].to(torch.float32) / scale).clamp_(-E4M3_MAX, E4M3_MAX)
        flat_out[s:e] = q.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes, scale


@dataclass
class DecodeInputs:
    q: torch.Tensor                  # [B, 64, 256] bf16
    k: torch.Tensor                  # contiguous [B, Lmax, 256] or paged [P, page, 256]; bf16 or uint8 (E4M3)
    v: torch.Tensor
    seq_lens: torch.Tensor           # [B] int32
    page_table: Optional[torch.Tensor] = None   # [B, max_pages] int32, or None
    page_size: int = 0
    kv_dtype: str = "bf16"           # "bf16" | "e4m3"
    k_scale: float = 1.0
    v_scale: float = 1.0
    softmax_scale: float = 1.0 / 16.0
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.to(torch.int64).sum().item())


def make_decode_inputs(seed: int, batch: int, seq_lens, *, lmax: Optional[int] = None,
                       page_size: int = 0, kv_dtype: str = "bf16") -> DecodeInputs:
    """Draw one decode-attention problem.

    seq_lens: an int (uniform length) or a sequence of per-sequence lengths.
    page_size > 0 gives a paged cache with a seeded random page placement.
    """
    g = torch.Generator().manual_seed(int(seed))
    if isinstance(seq_lens, int):
        lens = torch.full((batch,), seq_lens, dtype=torch.int32)
    else:
        lens = torch.as_tensor(list(seq_lens), dtype=torch.int32)
    assert lens.numel() == batch
    q = _randn_bf16(g, (batch, H, D))
    pt = None
    if page_size > 0:
        pages_per_seq = [(int(L) + page_size - 1) // page_size for L in lens.tolist()]
        pool = sum(pages_per_seq)
        max_pages = max([1] + pages_per_seq)
        perm = torch.randperm(max(pool, 1), generator=g)[:pool]
        pt = torch.full((batch, max_pages), -1, dtype=torch.int32)
        idx = 0
        for b, n in enumerate(pages_per_seq):
            if n:
                pt[b, :n] = perm[idx: idx + n].to(torch.int32)
            idx += n
        shape = (max(pool, 1), page_size, D)
    else:
        L = int(lmax if lmax is not None else max([1] + lens.tolist()))
        shape = (batch, L, D)
    k = _randn_bf16(g, shape)
    v = _randn_bf16(g, shape)
    k_scale = v_scale = 1.0
    if kv_dtype == "e4m3":
        k, k_scale = quantize_e4m3(k)
        v, v_scale = quantize_e4m3(v)
        fill = E4M3_NAN
    else:
        fill = float("nan")
    # Poison every cached row that lies past its sequence's length.
    for b, L in enumerate(lens.tolist()):
        if page_size > 0:
            n = (L + page_size - 1) // page_size
            if n and L % page_size:
                last = int(pt[b, n - 1])
                k[last, L % page_size:] = fill
                v[last, L % page_size:] = fill
        elif L < shape[1]:
            k[b, L:] = fill
            v[b, L:] = fill
    return DecodeInputs(q=q, k=k, v=v, seq_lens=lens, page_table=pt, page_size=page_size,
                        kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale,
                        meta={"seed": seed})


@dataclass
class ProjInputs:
    x: torch.Tensor      # [B, 7168] bf16
    w_qa: torch.Tensor   # [7168, 2048] bf16
    w_qb: torch.Tensor   # [2048, 64*256] bf16


def make_proj_inputs(seed: int, batch: int, hidden: int = HIDDEN, rank: int = RANK,
                     out_features: int = H * D) -> ProjInputs:
    g = torch.Generator().manual_seed(int(seed))
    x = _randn_bf16(g, (batch, hidden))
    w_qa = _randn_bf16(g, (hidden, rank), std=0.02)
    w_qb = _randn_bf16(g, (rank, out_features), std=0.02)
    return ProjInputs(x=x, w_qa=w_qa, w_qb=w_qb)


@dataclass
class KvAppendInputs:
    x: torch.Tensor    # [B, hidden] bf16 hidden states of the new tokens
    w_k: torch.Tensor  # [hidden, 256] bf16
    w_v: torch.Tensor  # [hidden, 256] bf16


def make_kv_append_inputs(seed: int, batch: int, hidden: int = HIDDEN) -> KvAppendInputs:
    """Hidden states ~ N(0, 1) and key/value weights ~ N(0, 0.02), as the projection's."""
    g = torch.Generator().manual_seed(int(seed))
    x = _randn_bf16(g, (batch, hidden))
    w_k = _randn_bf16(g, (hidden, D), std=0.02)
    w_v = _randn_bf16(g, (hidden, D), std=0.02)
    return KvAppendInputs(x=x, w_k=w_k, w_v=w_v)


@dataclass
class OutProjInputs:
    o: torch.Tensor    # [B, 64 * 256] bf16 attention outputs (heads x dim)
    w_o: torch.Tensor  # [64 * 256, hidden] bf16


def make_out_proj_inputs(seed: int, batch: int, hidden: int = HIDDEN) -> OutProjInputs:
    """Attention outputs ~ N(0, 1) and W_o ~ N(0, 0.02), as the projection's weights."""
    g = torch.Generator().manual_seed(int(seed))
    o = _randn_bf16(g, (batch, H * D))
    w_o = _randn_bf16(g, (H * D, hidden), std=0.02)
    return OutProjInputs(o=o, w_o=w_o)


@dataclass
class LseMergeInputs:
    o_parts: torch.Tensor    # [S, B, 64, 256] float32
    lse_parts: torch.Tensor  # [S, B, 64] float32, -inf marks an empty part


def make_lse_merge_inputs(seed: int, parts: int, batch: int, empty: float = 0.0,
                          lse_std: float = 4.0) -> LseMergeInputs:
    """Parts of a log-sum-exp merge: outputs ~ N(0, 1), lse ~ N(0, lse_std); a
    seeded fraction ``empty`` of the (part, sequence, head) entries is empty
    (lse = -inf, its output NaN, which must not reach the result)."""
    g = torch.Generator().manual_seed(int(seed))
    o = torch.randn((parts, batch, H, D), generator=g, dtype=torch.float32)
    lse = torch.randn((parts, batch, H), generator=g, dtype=torch.float32) * lse_std
    if empty > 0:
        hole = torch.rand((parts, batch, H), generator=g) < empty
        lse[hole] = float("-inf")
        o[hole] = float("nan")
    return LseMergeInputs(o_parts=o, lse_parts=lse)


# Grouped-query comparison shape (the Step-3 summary page, "Key points ->
# Ablations", compares MFA's decode latency with GQA's): 64 query heads of
# dimension 128 in 2 groups of 32, each group with its own key and value head
# of dimension 128, so a cached token costs 2 x 2 x 128 x 2 B = 1024 B, the same
# as MFA's one 256-wide key head and value head.
GQA_HEADS = 64
GQA_GROUPS = 2
GQA_DIM = 128


@dataclass
class GqaInputs:
    q: torch.Tensor                  # [B, 64, 128] bf16
    k: torch.Tensor                  # contiguous [B, Lmax, 2, 128] or paged [P, page, 2, 128]; bf16
    v: torch.Tensor
    seq_lens: torch.Tensor           # [B] int32
    page_table: Optional[torch.Tensor] = None
    page_size: int = 0
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(GQA_DIM)

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.sum())


def make_gqa_inputs(seed: int, batch: int, seq_lens, *, lmax: Optional[int] = None,
                    page_size: int = 0) -> GqaInputs:
    """One grouped-query problem, drawn like make_decode_inputs (q, K, V ~ N(0, 1)
    in bf16, seeded page placement, rows past a sequence's length NaN)."""
    g = torch.Generator().manual_seed(int(seed))
    if isinstance(seq_lens, int):
        lens = torch.full((batch,), seq_lens, dtype=torch.int32)
    else:
        lens = torch.as_tensor(list(seq_lens), dtype=torch.int32)
    assert lens.numel() == batch
    q = _randn_bf16(g, (batch, GQA_HEADS, GQA_DIM))
    pt = None
    if page_size > 0:
        pages_per_seq = [(int(L) + page_size - 1) // page_size for L in lens.tolist()]
        pool = sum(pages_per_seq)
        max_pages = max([1] + pages_per_seq)
        perm = torch.randperm(max(pool, 1), generator=g)[:pool]
        pt = torch.full((batch, max_pages), -1, dtype=torch.int32)
        idx = 0
        for b, n in enumerate(pages_per_seq):
            if n:
                pt[b, :n] = perm[idx: idx + n].to(torch.int32)
            idx += n
        shape = (max(pool, 1), page_size, GQA_GROUPS, GQA_DIM)
    else:
        L = int(lmax if lmax is not None else max([1] + lens.tolist()))
        shape = (batch, L, GQA_GROUPS, GQA_DIM)
    k = _randn_bf16(g, shape)
    v = _randn_bf16(g, shape)
    for b, L in enumerate(lens.tolist()):
        if page_size > 0:
            n = (L + page_size - 1) // page_size
            if n and L % page_size:
                last = int(pt[b, n - 1])
                k[last, L % page_size:] = float("nan")
                v[last, L % page_size:] = float("nan")
        elif L < shape[1]:
            k[b, L:] = float("nan")
            v[b, L:] = float("nan")
    return GqaInputs(q=q, k=k, v=v, seq_lens=lens, page_table=pt, page_size=page_size,
                     meta={"seed": seed})


GQA_WORKLOAD = dict(name="gqa_decode_b64_l4096_g2x128_bf16", batch=64, seq_len=4096)


def make_gqa_workload() -> GqaInputs:
    """The grouped-query comparison workload at the headline's size and bytes."""
    w = GQA_WORKLOAD
    inp = make_gqa_inputs(1100, w["batch"], w["seq_len"])
    inp.meta.update(name=w["name"])
    return inp


# The five workloads (seed = 1000 + index). Index 2 is the headline workload.
WORKLOADS = {
    1: dict(name="mfa_decode_b1_l512_bf16", batch=1, seq_len=512),
    2: dict(name="mfa_decode_b64_l4096_bf16", batch=64, seq_len=4096),
    3: dict(name="mfa_paged_decode_b256_l1024-8192_p64_bf16", batch=256, seq_len=(1024, 8192),
            page_size=64),
    # uniform lengths, batch below the SM count: one CTA per sequence (no
    # partials to merge) is the caller's split here
    4: dict(name="mfa_decode_b128_l4096_e4m3", batch=128, seq_len=4096, kv_dtype="e4m3",
            num_splits=1),
    5: dict(name="mfa_qproj_then_decode_b8_l65536_split16_bf16", batch=8, seq_len=65536,
            num_splits=16, qproj=True),
}


def workload_lengths(index: int) -> torch.Tensor:
    w = WORKLOADS[index]
    if isinstance(w["seq_len"], tuple):
        lo, hi = w["seq_len"]
        g = torch.Generator().manual_seed(5000 + index)
        return torch.randint(lo, hi + 1, (w["batch"],), generator=g, dtype=torch.int32)
    return torch.full((w["batch"],), w["seq_len"], dtype=torch.int32)


def make_workload(index: int):
    """Inputs of one of the five workloads: (DecodeInputs, ProjInputs or None)."""
    w = WORKLOADS[index]
    lens = workload_lengths(index)
    dec = make_decode_inputs(1000 + index, w["batch"], lens.tolist(),
                             page_size=w.get("page_size", 0), kv_dtype=w.get("kv_dtype", "bf16"))
    dec.meta.update(name=w["name"], num_splits=w.get("num_splits", 0))
    proj = make_proj_inputs(2000 + index, w["batch"]) if w.get("qproj") else None
    return dec, proj


def bits(t: torch.Tensor):
    """numpy view of a tensor's bit pattern (bf16 -> uint16, uint8 stays uint8)."""
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).numpy().view("uint16")
    return t.contiguous().numpy()
