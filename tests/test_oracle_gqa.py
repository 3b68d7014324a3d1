"""Pins of the oracle's grouped-query attention (GQA), the comparison shape for
MFA (the Step-3 summary page, "Key points -> Ablations": MFA beats GQA in
latency). The definition: H query heads in G groups of H / G consecutive heads,
group g attending over its own key and value head.

Each pin ties the C oracle to something other than itself: a NumPy restatement
that groups heads by reshaping, the already-pinned MFA (one shared head) oracle
applied group by group, a 50-digit decimal evaluation, closed forms, and
group isolation; planted group-mapping mistakes must fail a pin.
"""
import decimal

import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from oracle import mfa_oracle_np as onp


def _bits(t):
    return gen.bits(t)


def _case(seed, lens, H=8, G=2, D=16, page_size=0):
    g = torch.Generator().manual_seed(seed)
    B = len(lens)
    q = torch.randn(B, H, D, generator=g).to(torch.bfloat16)
    if page_size:
        inp = gen.make_gqa_inputs(seed, B, lens, page_size=page_size)
        return inp
    L = max(lens)
    k = torch.randn(B, L, G, D, generator=g).to(torch.bfloat16)
    v = torch.randn(B, L, G, D, generator=g).to(torch.bfloat16)
    return q, k, v, np.asarray(lens, np.int32)


def test_c_oracle_matches_numpy_twin(oracle_mod):
    q, k, v, lens = _case(1, [5, 17, 1, 0])
    out, lse = oracle_mod.gqa_decode(_bits(q), _bits(k), _bits(v), lens, 0.3)
    out2, lse2 = onp.gqa_decode(_bits(q), _bits(k), _bits(v), lens, 0.3)
    np.testing.assert_allclose(out, out2, rtol=1e-12, atol=1e-13)
    fin = np.isfinite(lse2)
    np.testing.assert_allclose(lse[fin], lse2[fin], rtol=1e-12, atol=1e-13)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse2))


def test_each_group_is_one_shared_head_attention(oracle_mod):
    """GQA is G independent MFA-style problems: the heads of group g over the
    cache's group-g rows equal the (separately pinned) shared-head oracle."""
    H, G, D = 8, 4, 16
    q, k, v, lens = _case(2, [9, 30, 2], H=H, G=G, D=D)
    out, lse = oracle_mod.gqa_decode(_bits(q), _bits(k), _bits(v), lens, 0.25)
    for g in range(G):
        heads = slice(g * H // G, (g + 1) * H // G)
        ref, lref = oracle_mod.decode(_bits(q[:, heads].contiguous()),
                                      _bits(k[:, :, g].contiguous()),
                                      _bits(v[:, :, g].contiguous()), lens, 0.25)
        np.testing.assert_allclose(out[:, heads], ref, rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[:, heads], lref, rtol=1e-13, atol=1e-14)


def test_groups_are_isolated(oracle_mod):
    """Changing group 1's keys and values leaves every group-0 head's output
    unchanged (bit for bit) and changes group 1's."""
    q, k, v, lens = _case(3, [12, 40])
    a, _ = oracle_mod.gqa_decode(_bits(q), _bits(k), _bits(v), lens, 0.3)
    k2, v2 = k.clone(), v.clone()
    k2[:, :, 1] = torch.flip(k[:, :, 1], dims=[1])
    v2[:, :, 1] = -v[:, :, 1]
    b, _ = oracle_mod.gqa_decode(_bits(q), _bits(k2), _bits(v2), lens, 0.3)
    assert np.array_equal(a[:, :4], b[:, :4])
    assert not np.allclose(a[:, 4:], b[:, 4:])


def test_single_token_returns_its_groups_value_row(oracle_mod):
    q, k, v, _ = _case(4, [1, 1])
    out, _ = oracle_mod.gqa_decode(_bits(q), _bits(k), _bits(v), np.array([1, 1], np.int32), 0.3)
    vf = onp.bf16_bits_to_f64(_bits(v))
    for h in range(8):
        assert np.array_equal(out[:, h], vf[:, 0, h // 4])


def test_paged_equals_contiguous(oracle_mod):
    lens = [1, 64, 65, 200]
    inp = gen.make_gqa_inputs(5, len(lens), lens, page_size=32)
    out_p, lse_p = oracle_mod.gqa_decode(_bits(inp.q), _bits(inp.k), _bits(inp.v),
                                         inp.seq_lens.numpy(), inp.softmax_scale,
                                         page_table=inp.page_table.numpy(), page_size=32)
    L = max(lens)
    kc = torch.zeros(len(lens), L, 2, 128, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for b, n in enumerate(lens):
        t = torch.arange(n)
        pages = inp.page_table[b, t // 32].long()
        kc[b, :n] = inp.k[pages, t % 32]
        vc[b, :n] = inp.v[pages, t % 32]
    out_c, lse_c = oracle_mod.gqa_decode(_bits(inp.q), _bits(kc), _bits(vc), inp.seq_lens.numpy(),
                                         inp.softmax_scale)
    assert np.array_equal(out_p, out_c) and np.array_equal(lse_p, lse_c)


def _decimal(qf, kf, vf, scale):
    decimal.getcontext().prec = 50
    Dd = decimal.Decimal
    s = [Dd(scale) * sum(Dd(a) * Dd(b) for a, b in zip(qf, kr)) for kr in kf]
    m = max(s)
    e = [(x - m).exp() for x in s]
    den = sum(e)
    return [float(sum(e[t] * Dd(vf[t][i]) for t in range(len(kf))) / den)
            for i in range(len(vf[0]))], float(m + den.ln())


def test_brute_force_decimal_on_tiny_inputs(oracle_mod):
    H, G, D = 4, 2, 4
    for seed, L in [(6, 1), (7, 3), (8, 6)]:
        q, k, v, lens = _case(seed, [L], H=H, G=G, D=D)
        out, lse = oracle_mod.gqa_decode(_bits(q), _bits(k), _bits(v), lens, 0.6)
        qf = onp.bf16_bits_to_f64(_bits(q))[0]
        kf = onp.bf16_bits_to_f64(_bits(k))[0]
        vf = onp.bf16_bits_to_f64(_bits(v))[0]
        for h in range(H):
            g = h // (H // G)
            ref, lref = _decimal(qf[h].tolist(), kf[:, g].tolist(), vf[:, g].tolist(), 0.6)
            np.testing.assert_allclose(out[0, h], ref, rtol=1e-14, atol=1e-15)
            assert abs(lse[0, h] - lref) <= 1e-14 * max(1.0, abs(lref))


def _mutant(kind):
    """The NumPy restatement with one planted mistake in the head-to-group map."""
    def gqa(q_bits, k, v, seq_lens, scale):
        q = onp.bf16_bits_to_f64(q_bits)
        kd, vd = onp.bf16_bits_to_f64(k), onp.bf16_bits_to_f64(v)
        B, H, D = q.shape
        G = kd.shape[2]
        out = np.zeros((B, H, D))
        for b in range(B):
            L = int(seq_lens[b])
            for h in range(H):
                g = (h % G) if kind == "interleaved_groups" else (h // (H // G))
                gk = (G - 1 - g) if kind == "value_group_swapped" else g
                s = scale * (kd[b, :L, g] @ q[b, h])
                w = np.exp(s - s.max())
                w /= w.sum()
                out[b, h] = w @ vd[b, :L, gk]
        return out
    return gqa


@pytest.mark.parametrize("kind", ["interleaved_groups", "value_group_swapped"])
def test_pins_catch_planted_group_mistakes(oracle_mod, kind):
    H, G, D = 8, 2, 16
    q, k, v, lens = _case(9, [7, 20], H=H, G=G, D=D)
    got = _mutant(kind)(_bits(q), _bits(k), _bits(v), lens, 0.3)
    failures = 0
    # pin: group by group, the shared-head oracle
    for g in range(G):
        heads = slice(g * H // G, (g + 1) * H // G)
        ref, _ = oracle_mod.decode(_bits(q[:, heads].contiguous()), _bits(k[:, :, g].contiguous()),
                                   _bits(v[:, :, g].contiguous()), lens, 0.3)
        failures += not np.allclose(got[:, heads], ref, rtol=1e-12, atol=1e-13)
    assert failures >= 1, f"planted mistake {kind!r} escaped the pin"
    # and the correct restatement passes the same pin
    good = onp.gqa_decode(_bits(q), _bits(k), _bits(v), lens, 0.3)[0]
    for g in range(G):
        heads = slice(g * H // G, (g + 1) * H // G)
        ref, _ = oracle_mod.decode(_bits(q[:, heads].contiguous()), _bits(k[:, :, g].contiguous()),
                                   _bits(v[:, :, g].contiguous()), lens, 0.3)
        np.testing.assert_allclose(good[:, heads], ref, rtol=1e-12, atol=1e-13)
