"""Pins for the float64 oracle, against facts the definition fixes.

No page prints a worked numerical example, so each part of the oracle is pinned
by something other than itself: closed forms (single token, identical keys,
zero scale, all-ones values), invariants (permutation of cached tokens, paged
vs. contiguous placement, split-and-merge), a 50-digit ``decimal`` evaluation of
the definition on tiny inputs, torch's independent E4M3 decoder, and the NumPy
twin as a second restatement. ``test_pins_catch_planted_mistakes`` plants
plausible mistakes in a copy of the NumPy restatement and checks that these pins
catch every one.
"""
import decimal
import math

import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from oracle import mfa_oracle_np as onp


def _bits(t):
    return gen.bits(t)


def _small(seed, B=3, lens=(5, 17, 1), lmax=20, H=4, D=8):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, D, generator=g).to(torch.bfloat16)
    k = torch.randn(B, lmax, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, lmax, D, generator=g).to(torch.bfloat16)
    return _bits(q), _bits(k), _bits(v), np.asarray(lens, np.int32)


def test_c_oracle_matches_numpy_twin(oracle_mod):
    for seed in range(4):
        q, k, v, lens = _small(seed)
        out_c, lse_c = oracle_mod.decode(q, k, v, lens, 0.37)
        out_n, lse_n = onp.decode(q, k, v, lens, 0.37)
        np.testing.assert_allclose(out_c, out_n, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse_c, lse_n, rtol=1e-12, atol=1e-14)


def test_single_token_returns_that_value_row_exactly(oracle_mod):
    q, k, v, _ = _small(1)
    lens = np.array([1, 1, 1], np.int32)
    out, lse = oracle_mod.decode(q, k, v, lens, 1.0 / 16)
    vrow = onp.bf16_bits_to_f64(v[:, 0, :])
    for h in range(q.shape[1]):
        assert np.array_equal(out[:, h, :], vrow)          # w = 1 exactly
    # lse of a single token is its own score
    s = (onp.bf16_bits_to_f64(q) * onp.bf16_bits_to_f64(k[:, 0, :])[:, None, :]).sum(-1) / 16
    np.testing.assert_allclose(lse, s, rtol=1e-14, atol=1e-15)


def test_identical_keys_give_mean_of_values(oracle_mod):
    q, k, v, _ = _small(2)
    k[:] = k[:, :1, :]                                    # every key row equal
    lens = np.array([5, 17, 20], np.int32)
    out, _ = oracle_mod.decode(q, k, v, lens, 0.5)
    vd = onp.bf16_bits_to_f64(v)
    for b, L in enumerate(lens):
        np.testing.assert_allclose(out[b], np.broadcast_to(vd[b, :L].mean(0), out[b].shape),
                                   rtol=1e-13, atol=1e-14)


def test_zero_scale_gives_mean_of_values(oracle_mod):
    q, k, v, lens = _small(3)
    out, _ = oracle_mod.decode(q, k, v, lens, 0.0)
    vd = onp.bf16_bits_to_f64(v)
    for b, L in enumerate(lens):
        np.testing.assert_allclose(out[b], np.broadcast_to(vd[b, :L].mean(0), out[b].shape),
                                   rtol=1e-13, atol=1e-14)


def test_weights_sum_to_one(oracle_mod):
    """With every value row all-ones, out = sum_t w_t, which must be 1."""
    q, k, v, lens = _small(4)
    one = _bits(torch.ones(1, dtype=torch.bfloat16))[0]
    v[:] = one
    out, _ = oracle_mod.decode(q, k, v, lens, 0.9)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-14)


def test_one_dominant_key_selects_its_value(oracle_mod):
    q, k, v, _ = _small(5, B=1, lens=(9,), lmax=9)
    j = 6
    # q_h = c * k_j with a large scale: softmax concentrates on token j
    kd = onp.bf16_bits_to_f64(k[0])
    qv = torch.tensor(np.broadcast_to(kd[j] * 4.0, (1, q.shape[1], q.shape[2])).copy(),
                      dtype=torch.float32).to(torch.bfloat16)
    out, _ = oracle_mod.decode(_bits(qv), k, v, np.array([9], np.int32), 64.0)
    np.testing.assert_allclose(out[0], np.broadcast_to(onp.bf16_bits_to_f64(v[0, j]), out[0].shape),
                               rtol=0, atol=1e-9)


def test_permuting_cached_tokens_leaves_output_unchanged(oracle_mod):
    q, k, v, _ = _small(6, B=1, lens=(20,), lmax=20)
    lens = np.array([20], np.int32)
    perm = np.random.default_rng(0).permutation(20)
    out1, lse1 = oracle_mod.decode(q, k, v, lens, 0.3)
    out2, lse2 = oracle_mod.decode(q, k[:, perm], v[:, perm], lens, 0.3)
    np.testing.assert_allclose(out1, out2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse1, lse2, rtol=1e-14, atol=1e-15)


def test_paged_placement_equals_contiguous(oracle_mod):
    """Same logical tokens, placed in shuffled pages: identical result."""
    lens = [37, 64, 1, 130]
    dec = gen.make_decode_inputs(7, 4, lens, page_size=16)
    # rebuild the contiguous slab from the page table
    lmax = max(lens)
    kc = torch.zeros(4, lmax, 256, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for b, L in enumerate(lens):
        for t in range(L):
            p = int(dec.page_table[b, t // 16])
            kc[b, t] = dec.k[p, t % 16]
            vc[b, t] = dec.v[p, t % 16]
    q = _bits(dec.q)
    sel = [(b, h) for b in range(4) for h in (0, 17, 63)]
    out_p, lse_p = oracle_mod.decode(q, _bits(dec.k), _bits(dec.v), dec.seq_lens.numpy(), 1 / 16,
                                     page_table=dec.page_table.numpy(), page_size=16, select=sel)
    out_c, lse_c = oracle_mod.decode(q, _bits(kc), _bits(vc), dec.seq_lens.numpy(), 1 / 16,
                                     select=sel)
    assert np.array_equal(out_p, out_c) and np.array_equal(lse_p, lse_c)


def test_split_and_merge_equals_unsplit(oracle_mod):
    q, k, v, _ = _small(8, B=1, lens=(20,), lmax=20)
    full, lse_full = oracle_mod.decode(q, k, v, np.array([20], np.int32), 0.4)
    cuts = [0, 3, 4, 11, 20]
    for h in range(q.shape[1]):
        parts, lses = [], []
        for a, e in zip(cuts[:-1], cuts[1:]):
            o, l = oracle_mod.decode(q, k[:, a:e], v[:, a:e], np.array([e - a], np.int32), 0.4)
            parts.append(o[0, h])
            lses.append(l[0, h])
        merged, lse = oracle_mod.combine(np.array(parts), np.array(lses))
        np.testing.assert_allclose(merged, full[0, h], rtol=1e-13, atol=1e-15)
        assert abs(lse - lse_full[0, h]) < 1e-13
    # an empty range carries no weight
    m2, _ = oracle_mod.combine(np.array([full[0, 0], np.zeros(full.shape[-1])]),
                               np.array([lse_full[0, 0], -np.inf]))
    np.testing.assert_array_equal(m2, full[0, 0])


def test_empty_sequence_gives_zeros_and_minus_inf(oracle_mod):
    q, k, v, _ = _small(9)
    out, lse = oracle_mod.decode(q, k, v, np.array([0, 3, 0], np.int32), 0.5)
    assert np.all(out[0] == 0) and np.all(out[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    assert np.all(np.isfinite(lse[1]))


def _decimal_attention(qf, kf, vf, scale):
    """The definition in 50-digit decimal arithmetic (independent of float64)."""
    decimal.getcontext().prec = 50
    D = decimal.Decimal
    s = [D(scale) * sum(D(a) * D(b) for a, b in zip(qf, kr)) for kr in kf]
    m = max(s)
    e = [(x - m).exp() for x in s]
    den = sum(e)
    out = [sum(e[t] * D(vf[t][i]) for t in range(len(kf))) / den for i in range(len(vf[0]))]
    lse = m + den.ln()
    return [float(x) for x in out], float(lse)


def test_brute_force_decimal_on_tiny_inputs(oracle_mod):
    for seed, L in [(10, 1), (11, 2), (12, 5), (13, 8)]:
        q, k, v, _ = _small(seed, B=1, lens=(L,), lmax=L, H=2, D=4)
        out, lse = oracle_mod.decode(q, k, v, np.array([L], np.int32), 0.7)
        qf = onp.bf16_bits_to_f64(q)[0]
        kf = onp.bf16_bits_to_f64(k)[0].tolist()
        vf = onp.bf16_bits_to_f64(v)[0].tolist()
        for h in range(2):
            ref, lref = _decimal_attention(qf[h].tolist(), kf, vf, 0.7)
            np.testing.assert_allclose(out[0, h], ref, rtol=1e-14, atol=1e-15)
            assert abs(lse[0, h] - lref) <= 1e-14 * max(1.0, abs(lref))


def test_e4m3_decode_all_codes(oracle_mod):
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine_c = np.array([oracle_mod.e4m3_to_double(c) for c in codes])
    mine_n = onp.e4m3_to_f64(codes)
    nan = np.isnan(ref)
    assert set(np.nonzero(nan)[0].tolist()) == {0x7F, 0xFF}
    assert np.array_equal(np.isnan(mine_c), nan) and np.array_equal(np.isnan(mine_n), nan)
    assert np.array_equal(mine_c[~nan], ref[~nan]) and np.array_equal(mine_n[~nan], ref[~nan])
    # spot values from the format: largest finite, smallest subnormal, one
    assert mine_c[0x7E] == 448.0 and mine_c[0x01] == 2.0 ** -9 and mine_c[0x38] == 1.0


def test_fp8_cache_uses_dequantised_values(oracle_mod):
    dec = gen.make_decode_inputs(14, 2, [7, 3], kv_dtype="e4m3")
    codes_k, codes_v = dec.k.numpy(), dec.v.numpy()
    lens = dec.seq_lens.numpy()
    q = _bits(dec.q)
    # unit scales: the E4M3 values are exact in float32, so a float32 cache holding
    # the decoded values must give the identical result
    kd = np.nan_to_num(onp.e4m3_to_f64(codes_k)).astype(np.float32)
    vd = np.nan_to_num(onp.e4m3_to_f64(codes_v)).astype(np.float32)
    out8, lse8 = oracle_mod.decode(q, codes_k, codes_v, lens, 1 / 16, kv_dtype=oracle_mod.E4M3)
    out32, lse32 = oracle_mod.decode(q, kd, vd, lens, 1 / 16, kv_dtype=oracle_mod.F32)
    assert np.array_equal(out8, out32) and np.array_equal(lse8, lse32)
    # k_scale multiplies every score: same as folding it into the softmax scale
    a, c = dec.k_scale, dec.v_scale
    out_k, _ = oracle_mod.decode(q, codes_k, codes_v, lens, 1 / 16, kv_dtype=oracle_mod.E4M3,
                                 k_scale=a)
    out_f, _ = oracle_mod.decode(q, codes_k, codes_v, lens, a / 16, kv_dtype=oracle_mod.E4M3)
    np.testing.assert_allclose(out_k, out_f, rtol=1e-13, atol=1e-15)
    # v_scale multiplies the output
    out_v, _ = oracle_mod.decode(q, codes_k, codes_v, lens, 1 / 16, kv_dtype=oracle_mod.E4M3,
                                 v_scale=c)
    np.testing.assert_allclose(out_v, c * out8, rtol=1e-13, atol=1e-15)
    # and the C oracle agrees with the NumPy restatement with both scales applied
    out_c, _ = oracle_mod.decode(q, codes_k, codes_v, lens, 1 / 16, kv_dtype=oracle_mod.E4M3,
                                 k_scale=a, v_scale=c)
    out_n, _ = onp.decode(q, codes_k, codes_v, lens, 1 / 16, kv_dtype=2, k_scale=a, v_scale=c)
    np.testing.assert_allclose(out_c, out_n, rtol=1e-12, atol=1e-14)


def test_query_projection_associativity_and_one_hot(oracle_mod):
    p = gen.make_proj_inputs(15, 3, hidden=64, rank=32, out_features=48)
    x, wa, wb = _bits(p.x), _bits(p.w_qa), _bits(p.w_qb)
    q = oracle_mod.query_proj(x, wa, wb)
    xf, waf, wbf = (onp.bf16_bits_to_f64(a) for a in (x, wa, wb))
    np.testing.assert_allclose(q, xf @ (waf @ wbf), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(q, onp.query_proj(x, wa, wb), rtol=1e-12, atol=1e-14)
    onehot = torch.zeros(2, 64, dtype=torch.bfloat16)
    onehot[0, 5] = 1.0
    onehot[1, 63] = 1.0
    q1 = oracle_mod.query_proj(_bits(onehot), wa, wb)
    np.testing.assert_allclose(q1[0], waf[5] @ wbf, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(q1[1], waf[63] @ wbf, rtol=1e-13, atol=1e-15)


def test_paged_oracle_rejects_out_of_range_page(oracle_mod):
    dec = gen.make_decode_inputs(16, 1, [20], page_size=16)
    pt = dec.page_table.numpy().copy()
    pt[0, 1] = 99
    with pytest.raises(ValueError):
        oracle_mod.decode(_bits(dec.q), _bits(dec.k), _bits(dec.v), dec.seq_lens.numpy(), 1 / 16,
                          page_table=pt, page_size=16)


# ---------------------------------------------------------------------------
# Planted mistakes: each mutant restates the definition with one plausible
# error; at least one of the pins above (re-run here against the mutant) fails.
# ---------------------------------------------------------------------------

def _mutant(kind):
    def decode(q_bits, k, v, seq_lens, scale):
        q = onp.bf16_bits_to_f64(q_bits)
        kd = onp.bf16_bits_to_f64(k)
        vd = onp.bf16_bits_to_f64(v)
        B, H, D = q.shape
        out = np.zeros((B, H, D))
        for b in range(B):
            L = int(seq_lens[b])
            Kb, Vb = kd[b, :L], vd[b, :L]
            sc = 1.0 if kind == "drop_scale" else scale
            s = sc * (q[b] @ Kb.T)
            if kind == "softmax_wrong_axis":
                e = np.exp(s - s.max(0, keepdims=True))
                w = e / e.sum(0, keepdims=True)
            else:
                e = np.exp(s - s.max(1, keepdims=True))
                w = e / (e.sum(1, keepdims=True) if kind != "no_normalise" else 1.0)
            if kind == "values_are_keys":
                Vb = Kb
            if kind == "off_by_one_length":
                w = w[:, :max(L - 1, 1)]
                Vb = Vb[:max(L - 1, 1)]
            if kind == "sign_flip":
                w = np.exp(-s) / np.exp(-s).sum(1, keepdims=True)
            out[b] = w @ Vb
        return out
    return decode


@pytest.mark.parametrize("kind", ["drop_scale", "softmax_wrong_axis", "no_normalise",
                                  "values_are_keys", "off_by_one_length", "sign_flip"])
def test_pins_catch_planted_mistakes(oracle_mod, kind):
    mut = _mutant(kind)
    failures = 0
    # pin: decimal brute force
    q, k, v, _ = _small(20, B=1, lens=(6,), lmax=6, H=2, D=4)
    out = mut(q, k, v, np.array([6], np.int32), 0.7)
    ref, _ = _decimal_attention(onp.bf16_bits_to_f64(q)[0, 0].tolist(),
                                onp.bf16_bits_to_f64(k)[0].tolist(),
                                onp.bf16_bits_to_f64(v)[0].tolist(), 0.7)
    failures += not np.allclose(out[0, 0], ref, rtol=1e-12, atol=1e-13)
    # pin: all-ones values
    q, k, v, lens = _small(21)
    one = _bits(torch.ones(1, dtype=torch.bfloat16))[0]
    v1 = v.copy()
    v1[:] = one
    failures += not np.allclose(mut(q, k, v1, lens, 0.9), 1.0, atol=1e-13)
    assert failures >= 1, f"planted mistake {kind!r} escaped every pin"
