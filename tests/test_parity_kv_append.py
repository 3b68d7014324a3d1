"""GPU parity of the new-token key/value projection and cache append
(``mfa_kv_append``) against the float64 oracle, through the C ABI.

The kernel accumulates in fp32 (split over the hidden dimension, partials summed
in a fixed order) and rounds once on store; the oracle rounds the exact float64
value. The two stored codes can therefore differ by one unit in the last place
when the exact value lies within the fp32 accumulation error of a rounding
boundary: every written element must match within one code step (same sign,
adjacent magnitude) and almost all must match exactly. Rows that are not
written must be untouched, bit for bit.
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa
from oracle import mfa_oracle_np as onp
from oracle import oracle as orc

from helpers import assert_close, decode_atol, oracle_decode, run_decode

pytestmark = pytest.mark.gpu


def _code_steps(a, b, fp8):
    """Distance in representable steps between two same-format code arrays."""
    a = a.astype(np.int64)
    b = b.astype(np.int64)
    sign = 0x80 if fp8 else 0x8000
    mag = sign - 1
    sa, sb = (a & sign) != 0, (b & sign) != 0
    ma, mb = a & mag, b & mag
    same = sa == sb
    # codes of one sign are ordered by magnitude; across signs count through zero
    return np.where(same, np.abs(ma - mb), ma + mb)


def _run(inp, k_cache, v_cache, pos, *, page_table=None, fp8=False, k_scale=1.0, v_scale=1.0):
    dev = "cuda"
    kc, vc = k_cache.clone().to(dev), v_cache.clone().to(dev)
    mfa.kv_append(inp.x.to(dev), inp.w_k.to(dev), inp.w_v.to(dev), kc, vc,
                  torch.as_tensor(pos, dtype=torch.int32, device=dev),
                  page_table=None if page_table is None else page_table.to(dev),
                  kv_dtype="e4m3" if fp8 else "bf16", k_scale=k_scale, v_scale=v_scale)
    status = mfa.read_status()
    return kc.cpu(), vc.cpu(), status


def _oracle(inp, k_cache, v_cache, pos, *, page_table=None, page_size=64, fp8=False,
            k_scale=1.0, v_scale=1.0):
    return orc.kv_append(gen.bits(inp.x), gen.bits(inp.w_k), gen.bits(inp.w_v),
                         gen.bits(k_cache), gen.bits(v_cache), np.asarray(pos, np.int32),
                         kv_dtype=orc.E4M3 if fp8 else orc.BF16,
                         page_table=None if page_table is None else page_table.numpy(),
                         page_size=page_size, k_scale=k_scale, v_scale=v_scale)


def _check(got_k, got_v, want_k, want_v, base_k, base_v, fp8, exact_frac=0.99):
    gk, gv = gen.bits(got_k), gen.bits(got_v)
    written = (want_k != base_k) | (want_v != base_v)
    # rows the append does not touch: identical to the input cache
    rows = written.reshape(-1, written.shape[-1]).any(-1)
    assert np.array_equal(gk.reshape(-1, gk.shape[-1])[~rows],
                          base_k.reshape(-1, base_k.shape[-1])[~rows])
    assert np.array_equal(gv.reshape(-1, gv.shape[-1])[~rows],
                          base_v.reshape(-1, base_v.shape[-1])[~rows])
    for g, w in ((gk, want_k), (gv, want_v)):
        g2 = g.reshape(-1, g.shape[-1])[rows]
        w2 = w.reshape(-1, w.shape[-1])[rows]
        steps = _code_steps(g2, w2, fp8)
        assert steps.max() <= 1, f"max step difference {steps.max()}"
        assert (steps == 0).mean() >= exact_frac, (steps == 0).mean()


def _bf16_cache(seed, shape):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


def _fp8_cache(seed, shape):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 0x70, shape, generator=g, dtype=torch.uint8)


def test_contiguous_bf16_small():
    inp = gen.make_kv_append_inputs(701, 5, hidden=256)
    kc, vc = _bf16_cache(1, (5, 40, 256)), _bf16_cache(2, (5, 40, 256))
    pos = [0, 7, 39, 13, 20]
    got_k, got_v, st = _run(inp, kc, vc, pos)
    assert st == 0
    want_k, want_v, _, _ = _oracle(inp, kc, vc, pos)
    _check(got_k, got_v, want_k, want_v, gen.bits(kc), gen.bits(vc), False)


@pytest.mark.parametrize("fp8", [False, True])
def test_paged_full_hidden(fp8):
    """The Step-3 hidden size (7168) and a 64-token paged cache."""
    B, ps, pages_per_seq = 6, 64, 3
    inp = gen.make_kv_append_inputs(702 + fp8, B, hidden=7168)
    npg = B * pages_per_seq
    shape = (npg, ps, 256)
    kc = _fp8_cache(3, shape) if fp8 else _bf16_cache(3, shape)
    vc = _fp8_cache(4, shape) if fp8 else _bf16_cache(4, shape)
    g = torch.Generator().manual_seed(5)
    table = torch.randperm(npg, generator=g).to(torch.int32).view(B, pages_per_seq)
    pos = [0, 63, 64, 191, 100, 130]
    ks, vs = (0.02, 0.03) if fp8 else (1.0, 1.0)
    got_k, got_v, st = _run(inp, kc, vc, pos, page_table=table, fp8=fp8, k_scale=ks, v_scale=vs)
    assert st == 0
    want_k, want_v, _, _ = _oracle(inp, kc, vc, pos, page_table=table, page_size=ps, fp8=fp8,
                                   k_scale=ks, v_scale=vs)
    _check(got_k, got_v, want_k, want_v, gen.bits(kc), gen.bits(vc), fp8,
           exact_frac=0.97 if fp8 else 0.99)


def test_decode_batch_contiguous_fp8():
    """A decode batch (64 sequences) appending into an E4M3 cache."""
    B, L = 64, 48
    inp = gen.make_kv_append_inputs(704, B, hidden=7168)
    kc, vc = _fp8_cache(6, (B, L, 256)), _fp8_cache(7, (B, L, 256))
    pos = [(7 * b) % L for b in range(B)]
    got_k, got_v, st = _run(inp, kc, vc, pos, fp8=True, k_scale=0.02, v_scale=0.02)
    assert st == 0
    want_k, want_v, _, _ = _oracle(inp, kc, vc, pos, fp8=True, k_scale=0.02, v_scale=0.02)
    _check(got_k, got_v, want_k, want_v, gen.bits(kc), gen.bits(vc), True, exact_frac=0.97)


def test_bad_position_is_reported_and_not_written():
    inp = gen.make_kv_append_inputs(705, 3, hidden=128)
    kc, vc = _bf16_cache(8, (3, 16, 256)), _bf16_cache(9, (3, 16, 256))
    got_k, got_v, st = _run(inp, kc, vc, [2, 16, 5])  # 16 is past the cache
    assert st == mfa.STATUS_CODES["MFA_ERR_BAD_INDEX"]
    want_k, want_v, _, _ = _oracle(inp, kc, vc, [2, 0, 5])
    assert np.array_equal(gen.bits(got_k)[1], gen.bits(kc)[1])
    assert np.array_equal(gen.bits(got_v)[1], gen.bits(vc)[1])
    for b in (0, 2):
        t = [2, 16, 5][b]
        assert _code_steps(gen.bits(got_k)[b, t], want_k[b, t], False).max() <= 1


def test_append_then_attend():
    """The appended row is the one the next decode-attention call reads."""
    B, L = 4, 300
    dec = gen.make_decode_inputs(706, B, [L] * B, lmax=L + 1)
    inp = gen.make_kv_append_inputs(707, B, hidden=512)
    pos = [L] * B
    got_k, got_v, st = _run(inp, dec.k, dec.v, pos)
    assert st == 0
    want_k, want_v, _, _ = _oracle(inp, dec.k, dec.v, pos)
    dec2 = gen.DecodeInputs(q=dec.q, k=got_k, v=got_v, seq_lens=torch.full((B,), L + 1,
                                                                          dtype=torch.int32))
    got = run_decode(dec2)
    ref, _ = oracle_decode(dec2)
    assert_close(got, ref, decode_atol(dec2, ref, torch.float32), "out")
