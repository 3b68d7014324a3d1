"""GPU parity of MFA decode attention (bf16 KV cache) against the float64 oracle,
through the C ABI. Every case compares every output element: small cases span
several 128-token tiles with ragged tails, and the full-size workloads run in
the launch configuration the benchmark times. The bound is 2e-3 on fp32
outputs at every sequence length (plus one bf16 rounding for bf16 outputs)."""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa

from helpers import (assert_close, decode_atol, max_err_by_length, oracle_decode, run_decode,
                     to_dev)

pytestmark = pytest.mark.gpu

RAGGED = [1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 300, 513]


def test_single_token_is_exact():
    dec = gen.make_decode_inputs(101, 5, [1, 1, 1, 1, 1])
    got = run_decode(dec)
    vrow = dec.v[:, 0, :].to(torch.float64).numpy()
    for h in range(64):
        assert np.array_equal(got[:, h, :], vrow)
    got16 = run_decode(dec, out_dtype=torch.bfloat16)
    assert np.array_equal(got16, got)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_ragged_contiguous_all_outputs(out_dtype):
    dec = gen.make_decode_inputs(102, len(RAGGED), RAGGED, lmax=520)
    got, lse = run_decode(dec, out_dtype=out_dtype, lse=True)
    ref, lref = oracle_decode(dec)
    print("max |err| by length:", {L: f"{e:.2e}" for L, e in max_err_by_length(dec, got, ref).items()})
    assert_close(got, ref, decode_atol(dec, ref, out_dtype), "out")
    assert_close(lse, lref, 1e-4 + 1e-5 * np.abs(lref), "lse")


def test_short_sequences_every_length():
    """Lengths 1..64, where a few tokens carry all of the softmax weight: the
    probabilities' precision decides the error here (2e-3 at every length)."""
    lens = list(range(1, 65))
    errs = {}
    for seed in (120, 121):
        dec = gen.make_decode_inputs(seed, len(lens), lens, lmax=64)
        got = run_decode(dec)
        ref, _ = oracle_decode(dec)
        for L, e in max_err_by_length(dec, got, ref).items():
            errs[L] = max(errs.get(L, 0.0), e)
        assert_close(got, ref, decode_atol(dec, ref, torch.float32), f"short, seed {seed}")
    print("max |err| by length:", {L: f"{e:.2e}" for L, e in errs.items()})


def test_concentrated_weights():
    """Two keys share almost all the weight (q aligned with both) and their
    values are far apart: rounding the probabilities to bf16 alone gives errors
    of several 1e-3 here (4.6e-3 at L = 2 in a float64 simulation of it)."""
    lens = [2, 3, 130, 1000]
    dec = gen.make_decode_inputs(122, len(lens), lens, lmax=1000)
    for b, L in enumerate(lens):
        k0 = dec.k[b, 0].float()
        k1 = dec.k[b, L - 1].float()
        dec.q[b] = ((k0 + k1) * (6.0 / 16.0)).to(torch.bfloat16)[None, :].expand(64, 256)
        dec.q[b, 1::2] = (dec.q[b, 1::2].float() * 1.001).to(torch.bfloat16)
        dec.v[b, 0] = (torch.sign(dec.v[b, 0].float()) * 4).to(torch.bfloat16)
        dec.v[b, L - 1] = -dec.v[b, 0]
    got = run_decode(dec)
    ref, _ = oracle_decode(dec)
    err = assert_close(got, ref, decode_atol(dec, ref, torch.float32), "concentrated")
    print(f"concentrated weights: max |err| {err:.2e}")


def test_plain_entry_point_matches_ex():
    dec = gen.make_decode_inputs(103, 6, [700, 1, 129, 4096, 0, 2000])
    a = run_decode(dec, plain=True)
    b = run_decode(dec)
    assert np.array_equal(a, b)
    ref, _ = oracle_decode(dec)
    assert_close(a, ref, decode_atol(dec, ref, torch.float32), "plain")


def test_identical_keys_give_mean_of_values():
    dec = gen.make_decode_inputs(104, 3, [77, 300, 1000])
    dec.k[:] = dec.k[:, :1, :]
    got = run_decode(dec)
    for b, L in enumerate(dec.seq_lens.tolist()):
        mean = dec.v[b, :L].to(torch.float64).mean(0).numpy()
        assert np.max(np.abs(got[b] - mean[None, :])) <= 2e-3


def test_empty_sequences_give_zeros_and_minus_inf():
    dec = gen.make_decode_inputs(105, 5, [0, 300, 0, 1, 0])
    got, lse = run_decode(dec, lse=True)
    for b in (0, 2, 4):
        assert np.all(got[b] == 0) and np.all(np.isneginf(lse[b]))
    ref, lref = oracle_decode(dec)
    assert_close(got, ref, decode_atol(dec, ref, torch.float32), "out")


@pytest.mark.parametrize("page_size", [16, 32, 64, 128, 256])
def test_paged_is_bit_exact_with_contiguous(page_size):
    lens = [1, 64, 65, 200, 513, 1000, 129, 4097]
    dec = gen.make_decode_inputs(106 + page_size, len(lens), lens, page_size=page_size)
    # the same logical rows laid out contiguously
    lmax = max(lens)
    kc = torch.zeros(len(lens), lmax, 256, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for b, L in enumerate(lens):
        t = torch.arange(L)
        pages = dec.page_table[b, t // page_size].long()
        kc[b, :L] = dec.k[pages, t % page_size]
        vc[b, :L] = dec.v[pages, t % page_size]
    cont = gen.DecodeInputs(q=dec.q, k=kc, v=vc, seq_lens=dec.seq_lens)
    got_p, lse_p = run_decode(dec, lse=True)
    got_c, lse_c = run_decode(cont, lse=True)
    assert np.array_equal(got_p, got_c)
    assert np.array_equal(lse_p, lse_c)
    ref, _ = oracle_decode(dec)
    assert_close(got_p, ref, decode_atol(dec, ref, torch.float32), "paged")


@pytest.mark.parametrize("num_splits", [1, 2, 3, 7, 16])
def test_fixed_splits(num_splits):
    lens = [5000, 129, 1, 2048, 0, 777]
    dec = gen.make_decode_inputs(107, len(lens), lens)
    got, lse = run_decode(dec, num_splits=num_splits, lse=True)
    ref, lref = oracle_decode(dec)
    assert_close(got, ref, decode_atol(dec, ref, torch.float32), f"splits={num_splits}")
    finite = np.isfinite(lref)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lref))
    assert_close(lse[finite], lref[finite], 1e-4 + 1e-5 * np.abs(lref[finite]), "lse")


def test_more_sequences_than_sms_and_many_short_ones():
    rng = np.random.default_rng(7)
    lens = rng.integers(0, 300, 400).tolist()
    dec = gen.make_decode_inputs(108, len(lens), lens)
    got = run_decode(dec)
    ref, _ = oracle_decode(dec)
    assert_close(got, ref, decode_atol(dec, ref, torch.float32), "many")


def test_strided_q_and_out():
    dec = gen.make_decode_inputs(109, 4, [300, 1, 5000, 64])
    t = to_dev(dec)
    qbig = torch.zeros(4, 64, 264, dtype=torch.bfloat16, device="cuda")
    qbig[:, :, :256] = t["q"]
    q = qbig[:, :, :256]
    outbig = torch.full((4, 66, 256), 7.0, dtype=torch.float32, device="cuda")
    out = outbig[:, 1:65, :]
    mfa.decode_attention_ex(q, t["k"], t["v"], None, t["seq_lens"], out, 1 / 16)
    assert mfa.read_status() == 0
    ref, _ = oracle_decode(dec)
    got = out.double().cpu().numpy()
    assert_close(got, ref, decode_atol(dec, ref, torch.float32), "strided")
    assert torch.all(outbig[:, 0] == 7.0) and torch.all(outbig[:, 65] == 7.0)


def test_repeat_calls_are_bitwise_deterministic():
    dec = gen.make_decode_inputs(110, 9, [4096, 3000, 17, 9000, 1, 128, 256, 640, 2222])
    t = to_dev(dec)
    a = run_decode(dec, tensors=t)
    b = run_decode(dec, tensors=t)
    assert np.array_equal(a, b)


def test_bad_page_index_is_reported_not_faulted():
    dec = gen.make_decode_inputs(111, 2, [100, 200], page_size=64)
    dec.page_table[1, 2] = 10_000
    t = to_dev(dec)
    out = torch.zeros(2, 64, 256, device="cuda")
    mfa.decode_attention_ex(t["q"], t["k"], t["v"], t["page_table"], t["seq_lens"], out, 1 / 16)
    assert mfa.read_status() == mfa.STATUS_CODES["MFA_ERR_BAD_INDEX"]
    assert mfa.read_status() == 0  # cleared by the previous read


def test_length_beyond_cache_is_reported():
    dec = gen.make_decode_inputs(112, 2, [100, 200], lmax=256)
    t = to_dev(dec)
    t["seq_lens"][1] = 257
    out = torch.zeros(2, 64, 256, device="cuda")
    mfa.decode_attention_ex(t["q"], t["k"], t["v"], None, t["seq_lens"], out, 1 / 16)
    assert mfa.read_status() == mfa.STATUS_CODES["MFA_ERR_BAD_INDEX"]


# ---- the workloads at full size, every output ------------------------------

def _full_workload_check(index, num_splits=0):
    dec, _ = gen.make_workload(index)
    got = run_decode(dec, num_splits=num_splits)
    assert np.all(np.isfinite(got))
    ref, _ = oracle_decode(dec)
    err = assert_close(got, ref, decode_atol(dec, ref, torch.float32), gen.WORKLOADS[index]["name"])
    print(f"{gen.WORKLOADS[index]['name']}: max |err| {err:.2e} over {got.size} outputs")
    return err


def test_workload1_all_outputs():
    _full_workload_check(1)


def test_workload2_all_outputs():
    _full_workload_check(2)


def test_workload3_paged_all_outputs():
    _full_workload_check(3)


def test_workload5_attention_split16_all_outputs():
    _full_workload_check(5, num_splits=16)
