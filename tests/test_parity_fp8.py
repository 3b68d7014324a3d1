"""GPU parity of MFA decode attention over an FP8 E4M3 KV cache with per-tensor
scales, against the float64 oracle on the dequantised cache, through the C ABI.

Tolerance: max |err| <= 3e-2 (the stated FP8-KV target) at every length. The
kernel runs E4M3 x E4M3 tensor-core products (kind::f8f6f4) straight from the
cache, with q and the probabilities entering as exact E4M3 pairs hi + lo, so
its error stays at the level of the bf16 path; the tests report it.
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa

from helpers import assert_close, decode_atol, max_err_by_length, oracle_decode, run_decode

pytestmark = pytest.mark.gpu

FP8_TOL = 3e-2


def test_every_e4m3_code_decodes_exactly():
    """One cached token: the output is that V row, i.e. the decoded codes."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    codes[0x7F] = 0   # the two NaN codes
    codes[0xFF] = 0
    dec = gen.make_decode_inputs(501, 1, [1], kv_dtype="e4m3")
    dec.v[0, 0] = codes
    dec.k_scale = dec.v_scale = 1.0
    got = run_decode(dec)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for h in range(64):
        assert np.array_equal(got[0, h], want), f"head {h}"
    # with a v_scale the output is code * scale (one float32 product)
    dec.v_scale = 0.375
    got = run_decode(dec)
    assert np.array_equal(got[0, 0], (want.astype(np.float32) * np.float32(0.375)).astype(np.float64))


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_fp8_ragged_contiguous(out_dtype):
    lens = [1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 300, 513, 4000]
    dec = gen.make_decode_inputs(502, len(lens), lens, lmax=4100, kv_dtype="e4m3")
    got, lse = run_decode(dec, out_dtype=out_dtype, lse=True)
    ref, lref = oracle_decode(dec)
    print("max |err| by length:", {L: f"{e:.2e}" for L, e in max_err_by_length(dec, got, ref).items()})
    err = assert_close(got, ref, decode_atol(dec, ref, out_dtype, base=FP8_TOL), "fp8 out")
    assert_close(lse, lref, 1e-4 + 1e-5 * np.abs(lref), "fp8 lse")
    assert err < FP8_TOL


@pytest.mark.parametrize("page_size,num_splits", [(16, 0), (64, 0), (256, 0), (64, 3)])
def test_fp8_paged_is_bit_exact_with_contiguous(page_size, num_splits):
    """Paged and contiguous caches give identical bits; num_splits = 3 (6 x 3 units,
    fewer than the CTAs) runs the one-q-buffer, five-slot FP8 kernels."""
    lens = [1, 65, 200, 1000, 4097, 129]
    dec = gen.make_decode_inputs(503 + page_size, len(lens), lens, page_size=page_size,
                                 kv_dtype="e4m3")
    lmax = max(lens)
    kc = torch.zeros(len(lens), lmax, 256, dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    for b, L in enumerate(lens):
        t = torch.arange(L)
        pages = dec.page_table[b, t // page_size].long()
        kc[b, :L] = dec.k[pages, t % page_size]
        vc[b, :L] = dec.v[pages, t % page_size]
    cont = gen.DecodeInputs(q=dec.q, k=kc, v=vc, seq_lens=dec.seq_lens, kv_dtype="e4m3",
                            k_scale=dec.k_scale, v_scale=dec.v_scale)
    got_p = run_decode(dec, num_splits=num_splits)
    got_c = run_decode(cont, num_splits=num_splits)
    assert np.array_equal(got_p, got_c)
    ref, _ = oracle_decode(dec)
    assert_close(got_p, ref, decode_atol(dec, ref, torch.float32, base=FP8_TOL), "fp8 paged")


def test_fp8_fixed_splits():
    lens = [5000, 129, 0, 2048]
    dec = gen.make_decode_inputs(510, len(lens), lens, kv_dtype="e4m3")
    got = run_decode(dec, num_splits=5)
    ref, _ = oracle_decode(dec)
    assert_close(got, ref, decode_atol(dec, ref, torch.float32, base=FP8_TOL), "fp8 splits")


def test_workload4_fp8_all_outputs():
    """Workload 4 at full size, in both launch configurations the benchmark
    times: the balanced plan and one CTA per sequence (num_splits = 1)."""
    dec, _ = gen.make_workload(4)
    ref, _ = oracle_decode(dec)
    tol = decode_atol(dec, ref, torch.float32, base=FP8_TOL)
    for splits in (0, dec.meta["num_splits"]):
        got = run_decode(dec, num_splits=splits)
        assert np.all(np.isfinite(got))
        err = assert_close(got, ref, tol, f"wl4 splits={splits}")
        print(f"workload 4 (num_splits={splits}): max |err| {err:.2e} over {got.size} outputs")
