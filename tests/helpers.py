"""Shared helpers for the parity tests: run the CUDA path through the binding,
run the oracle on the same inputs, and the tolerances used to compare them.

Tolerances (floating point; integer/index work is compared bit-exactly):
  * bf16 KV cache, fp32 output: max |err| <= 2e-3 on unit-scale outputs (the
    target stated for this operation). The kernel rounds softmax probabilities to
    bf16 (relative 2^-9) before the PV product, which bounds its error by
    2^-9 * max_t |V[t]|; for very short sequences (L < 64) whose outputs are not
    averaged down that bound can exceed 2e-3, so there the tolerance is
    max(2e-3, 2^-8 * max_t |V[t]|).
  * bf16 output adds the output rounding, 2^-8 * |ref|.
  * lse: 1e-4 + 1e-5 |lse| (fp32 row sums, hardware exp2/log2).
  * query projection: 2^-8 |ref| (one bf16 rounding of the result) plus
    1e-4 * max |ref| for fp32 accumulation.
"""
from __future__ import annotations

import numpy as np
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa
from oracle import oracle as orc


def to_dev(dec: gen.DecodeInputs):
    dev = "cuda"
    return dict(q=dec.q.to(dev), k=dec.k.to(dev), v=dec.v.to(dev),
                seq_lens=dec.seq_lens.to(dev),
                page_table=None if dec.page_table is None else dec.page_table.to(dev))


def run_decode(dec: gen.DecodeInputs, *, out_dtype=torch.float32, num_splits=0, lse=False,
               plain=False, tensors=None):
    t = tensors or to_dev(dec)
    B = dec.batch
    out = torch.full((B, 64, 256), float("nan"), dtype=out_dtype, device="cuda")
    lse_out = torch.full((B, 64), float("nan"), dtype=torch.float32, device="cuda") if lse else None
    if plain:
        mfa.decode_attention(t["q"], t["k"], t["v"], t["page_table"], t["seq_lens"], out,
                             dec.softmax_scale, dec.kv_dtype)
    else:
        mfa.decode_attention_ex(t["q"], t["k"], t["v"], t["page_table"], t["seq_lens"], out,
                                dec.softmax_scale, dec.kv_dtype, k_scale=dec.k_scale,
                                v_scale=dec.v_scale, num_splits=num_splits, lse_out=lse_out)
    status = mfa.read_status()
    assert status == 0, f"device status {mfa.STATUS.get(status, status)}"
    res = out.float().cpu().numpy().astype(np.float64)
    if lse:
        return res, lse_out.cpu().numpy().astype(np.float64)
    return res


def oracle_decode(dec: gen.DecodeInputs, select=None):
    kvd = orc.E4M3 if dec.kv_dtype == "e4m3" else orc.BF16
    pt = None if dec.page_table is None else dec.page_table.numpy()
    return orc.decode(gen.bits(dec.q), gen.bits(dec.k), gen.bits(dec.v), dec.seq_lens.numpy(),
                      dec.softmax_scale, kv_dtype=kvd, page_table=pt,
                      page_size=dec.page_size or 64, k_scale=dec.k_scale, v_scale=dec.v_scale,
                      select=select)


def v_absmax_per_seq(dec: gen.DecodeInputs) -> np.ndarray:
    """max_t |V_b[t]| over each sequence's valid rows (dequantised)."""
    out = np.zeros(dec.batch)
    v = dec.v
    for b, L in enumerate(dec.seq_lens.tolist()):
        if L == 0:
            continue
        if dec.page_table is None:
            rows = v[b, :L]
        else:
            t = torch.arange(L)
            rows = v[dec.page_table[b, t // dec.page_size].long(), t % dec.page_size]
        if dec.kv_dtype == "e4m3":
            vals = rows.view(torch.float8_e4m3fn).to(torch.float64) * dec.v_scale
        else:
            vals = rows.to(torch.float64)
        out[b] = float(vals.abs().max())
    return out


def decode_atol(dec: gen.DecodeInputs, ref: np.ndarray, out_dtype, base=2e-3, b_index=None):
    """Per-element absolute tolerance, broadcastable to ref ([B,H,D] or [n,D])."""
    vmax = v_absmax_per_seq(dec)
    lens = dec.seq_lens.numpy()
    per_b = np.where(lens < 64, np.maximum(base, 2.0 ** -8 * vmax), base)
    if b_index is not None:
        tol = per_b[np.asarray(b_index)][:, None]
    else:
        tol = per_b[:, None, None]
    tol = np.broadcast_to(tol, ref.shape).copy()
    if out_dtype == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    return tol


def assert_close(got, ref, atol, what=""):
    err = np.abs(got - ref)
    bad = ~(err <= atol)
    if bad.any():
        idx = np.argwhere(bad)[0]
        raise AssertionError(
            f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; first at {tuple(idx)}: "
            f"got {got[tuple(idx)]!r} ref {ref[tuple(idx)]!r} atol {atol[tuple(idx)]!r}; "
            f"max err {np.nanmax(err):.3e}")
    return float(np.max(err)) if err.size else 0.0


def sample_pairs(B, n, seed):
    rng = np.random.default_rng(seed)
    bs = rng.integers(0, B, n)
    hs = rng.integers(0, 64, n)
    pairs = sorted(set(zip(bs.tolist(), hs.tolist())))
    return pairs
