"""Pins for the oracle's new-token key/value projection and cache append, and for its
output projection.

The rounding functions are pinned by hand-computed ties and landmarks of the
formats (bf16: binary32's top half; E4M3: the OCP FP8 definition, largest
finite 448, smallest subnormal 2^-9), by round-trips of every finite code, and by
torch's independent float32 conversions on values exact in float32. The
projection is pinned by one-hot weights (exact selection) and the NumPy twin;
the append by placement invariants (paged equals contiguous, untouched rows stay
as they were).
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from oracle import mfa_oracle_np as onp


def test_bf16_round_ties_and_landmarks(oracle_mod):
    o = oracle_mod
    assert o.bf16_round(1.0) == 0x3F80
    assert o.bf16_round(1 + 2 ** -8) == 0x3F80  # halfway between 1 and 1 + 2^-7: even
    assert o.bf16_round(1 + 3 * 2 ** -8) == 0x3F82  # halfway: even
    assert o.bf16_round(1 + 2 ** -8 + 2 ** -30) == 0x3F81  # just past halfway
    assert o.bf16_round(-2.5) == 0xC020
    assert o.bf16_round(2 ** -133) == 0x0001  # smallest subnormal
    assert o.bf16_round(3 * 2 ** -134) == 0x0002  # halfway between 1 and 2 quanta: even
    assert o.bf16_round(0.0) == 0x0000 and o.bf16_round(-0.0) == 0x8000
    assert o.bf16_round(2.0 ** 128) == 0x7F80


def test_bf16_round_fixes_every_bf16_and_matches_torch():
    from oracle import oracle as o
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 0x7F80, 3000).astype(np.uint16)
    bits = np.concatenate([bits, bits | 0x8000]).astype(np.uint16)
    vals = onp.bf16_bits_to_f64(bits)
    assert all(o.bf16_round(v) == int(b) for v, b in zip(vals, bits))
    f = rng.standard_normal(3000).astype(np.float32) * np.float32(37.0)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    mine = np.array([o.bf16_round(float(v)) for v in f], np.uint16)
    assert np.array_equal(mine, ref)


def test_e4m3_encode_ties_saturation_and_round_trip(oracle_mod):
    o = oracle_mod
    assert o.e4m3_encode(1.0) == 0x38 and o.e4m3_encode(-1.0) == 0xB8
    assert o.e4m3_encode(448.0) == 0x7E and o.e4m3_encode(1e4) == 0x7E
    assert o.e4m3_encode(-1e4) == 0xFE
    assert o.e4m3_encode(2 ** -9) == 0x01 and o.e4m3_encode(2 ** -10) == 0x00  # tie: even
    assert o.e4m3_encode(3 * 2 ** -10) == 0x02  # halfway between 1 and 2 quanta: even
    assert o.e4m3_encode(1.0625) == 0x38 and o.e4m3_encode(1.1875) == 0x3A  # ties: even
    for code in range(256):
        if code & 0x7F == 0x7F:
            continue
        assert o.e4m3_encode(o.e4m3_to_double(code)) == code


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    rng = np.random.default_rng(8)
    f = (rng.standard_normal(3000) * 40.0).clip(-440, 440).astype(np.float32)
    ref = torch.from_numpy(f).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle_mod.e4m3_encode(float(v)) for v in f], np.uint8)
    assert np.array_equal(mine, ref)


def test_kv_projection_one_hot_and_twin(oracle_mod):
    g = torch.Generator().manual_seed(9)
    x = torch.randn(3, 64, generator=g).to(torch.bfloat16)
    perm = torch.randperm(64, generator=g)[:16]
    wk = torch.zeros(64, 16, dtype=torch.bfloat16)
    wv = torch.zeros(64, 16, dtype=torch.bfloat16)
    wk[perm, torch.arange(16)] = 1.0
    wv[perm, torch.arange(16)] = -2.0
    k, v = oracle_mod.kv_project(gen.bits(x), gen.bits(wk), gen.bits(wv))
    xf = x.double().numpy()
    assert np.array_equal(k, xf[:, perm.numpy()])
    assert np.array_equal(v, -2.0 * xf[:, perm.numpy()])
    wk2 = torch.randn(64, 16, generator=g).to(torch.bfloat16)
    wv2 = torch.randn(64, 16, generator=g).to(torch.bfloat16)
    kc, vc = oracle_mod.kv_project(gen.bits(x), gen.bits(wk2), gen.bits(wv2))
    kn, vn = onp.kv_project(gen.bits(x), gen.bits(wk2), gen.bits(wv2))
    np.testing.assert_allclose(kc, kn, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(vc, vn, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("kv_dtype", ["bf16", "e4m3"])
def test_kv_append_placement(oracle_mod, kv_dtype):
    g = torch.Generator().manual_seed(10)
    B, Dm, D, L, ps = 3, 64, 8, 12, 4
    x = gen.bits(torch.randn(B, Dm, generator=g).to(torch.bfloat16))
    wk = gen.bits(torch.randn(Dm, D, generator=g).to(torch.bfloat16))
    wv = gen.bits(torch.randn(Dm, D, generator=g).to(torch.bfloat16))
    pos = np.array([0, 5, 11], np.int32)
    e4 = kv_dtype == "e4m3"
    dt = np.uint8 if e4 else np.uint16
    rng = np.random.default_rng(11)
    kc = rng.integers(0, 0x70 if e4 else 0x3F00, (B, L, D)).astype(dt)
    vc = rng.integers(0, 0x70 if e4 else 0x3F00, (B, L, D)).astype(dt)
    kw = dict(kv_dtype=oracle_mod.E4M3 if e4 else oracle_mod.BF16, k_scale=0.5, v_scale=0.25)
    k_new, v_new, k, v = oracle_mod.kv_append(x, wk, wv, kc, vc, pos, **kw)
    for b in range(B):
        t = pos[b]
        rest = [i for i in range(L) if i != t]
        assert np.array_equal(k_new[b, rest], kc[b, rest]) and np.array_equal(v_new[b, rest], vc[b, rest])
        want_k = [oracle_mod.e4m3_encode(val / 0.5) if e4 else oracle_mod.bf16_round(val) for val in k[b]]
        want_v = [oracle_mod.e4m3_encode(val / 0.25) if e4 else oracle_mod.bf16_round(val) for val in v[b]]
        assert list(k_new[b, t]) == want_k and list(v_new[b, t]) == want_v
    # the same rows through a page table land at the same logical positions
    npg = B * L // ps
    perm = rng.permutation(npg).astype(np.int32)
    table = perm.reshape(B, L // ps)
    kp = np.zeros((npg, ps, D), dt)
    vp = np.zeros((npg, ps, D), dt)
    for b in range(B):
        for t in range(L):
            kp[table[b, t // ps], t % ps] = kc[b, t]
            vp[table[b, t // ps], t % ps] = vc[b, t]
    kp_new, vp_new, _, _ = oracle_mod.kv_append(x, wk, wv, kp, vp, pos, page_table=table,
                                                page_size=ps, **kw)
    for b in range(B):
        for t in range(L):
            assert np.array_equal(kp_new[table[b, t // ps], t % ps], k_new[b, t])
            assert np.array_equal(vp_new[table[b, t // ps], t % ps], v_new[b, t])
    with pytest.raises(ValueError):
        oracle_mod.kv_append(x, wk, wv, kc, vc, np.array([0, 5, L], np.int32), **kw)


def test_output_projection_one_hot_twin_and_decimal(oracle_mod):
    """The output projection oracle: one-hot rows select weight rows exactly, it
    agrees with the NumPy twin, and a 50-digit evaluation on a tiny case."""
    import decimal
    g = torch.Generator().manual_seed(12)
    o = torch.randn(3, 128, generator=g).to(torch.bfloat16)
    w = torch.randn(128, 48, generator=g).to(torch.bfloat16)
    y = oracle_mod.out_proj(gen.bits(o), gen.bits(w))
    np.testing.assert_allclose(y, onp.out_proj(gen.bits(o), gen.bits(w)), rtol=1e-12, atol=1e-13)
    onehot = torch.zeros(2, 128, dtype=torch.bfloat16)
    onehot[0, 3] = 1.0
    onehot[1, 127] = -4.0
    y1 = oracle_mod.out_proj(gen.bits(onehot), gen.bits(w))
    wf = w.double().numpy()
    assert np.array_equal(y1[0], wf[3]) and np.array_equal(y1[1], -4.0 * wf[127])
    decimal.getcontext().prec = 50
    of, wf2 = o.double().numpy(), w.double().numpy()
    for b, n in ((0, 0), (2, 47), (1, 20)):
        exact = sum(decimal.Decimal(float(of[b, k])) * decimal.Decimal(float(wf2[k, n]))
                    for k in range(128))
        assert abs(float(exact) - y[b, n]) <= 1e-12 * max(1.0, abs(float(exact)))
