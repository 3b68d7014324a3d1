"""Shared helpers for the parity tests: run the CUDA path through the binding,
run the oracle on the same inputs, and the tolerances used to compare them.

Tolerances (floating point; integer/index work is compared bit-exactly):
  * bf16 KV cache, fp32 output: max |err| <= 2e-3 at every sequence length (the
    target stated for this operation on unit-scale outputs). The kernel carries
    the softmax probabilities into the PV product as a bf16 pair hi + lo
    (~16 significant bits), so its error is far below that bound even where a
    few tokens carry all the weight.
  * FP8 (E4M3) KV cache: max |err| <= 3e-2 against the oracle on the
    dequantised cache.
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


def decode_atol(dec: gen.DecodeInputs, ref: np.ndarray, out_dtype, base=2e-3, b_index=None):
    """Per-element absolute tolerance, the shape of ref ([B,H,D] or [n,D]): `base`
    everywhere, plus one bf16 rounding of the result for bf16 outputs."""
    tol = np.full(ref.shape, base)
    if out_dtype == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    return tol


def max_err_by_length(dec: gen.DecodeInputs, got: np.ndarray, ref: np.ndarray) -> dict:
    """{sequence length: max |got - ref| over its outputs} (reported by the tests)."""
    out = {}
    for b, L in enumerate(dec.seq_lens.tolist()):
        e = float(np.max(np.abs(got[b] - ref[b])))
        out[L] = max(out.get(L, 0.0), e)
    return out


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
