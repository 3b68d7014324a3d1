"""The allocation-free decode entry point, mfa_decode_attention_noalloc.

Some callers cannot allocate device memory when they call in: a host framework
that owns every device allocation through its own pool, or a latency-critical
loop that must not pay cudaMalloc's cost and implicit synchronisation. For them
the library keeps the split workspace in a fixed device array of its own.

These tests call that entry point through the C ABI twice in a row and check
both results against the workspace-taking entry point
(mfa_decode_attention_ex), within the decode tolerance the parity tests use.
They pass run alone in a fresh process or after the rest of the suite.
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa

from helpers import assert_close, decode_atol, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(t, dec, out, lse=None, num_splits=0):
    """Direct C-ABI call of mfa_decode_attention_noalloc; returns the status code."""
    return mfa.lib().mfa_decode_attention_noalloc(
        mfa.describe(t["q"]), mfa.describe(t["k"]), mfa.describe(t["v"]),
        mfa.describe(t["page_table"]), mfa.describe(t["seq_lens"]), mfa.describe(out),
        float(dec.softmax_scale), mfa.MFA_BF16, 1.0, 1.0, int(num_splits), mfa.describe(lse),
        torch.cuda.current_stream().cuda_stream)


def _reference(t, dec, num_splits=0):
    B = dec.batch
    out = torch.empty(B, 64, 256, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, 64, dtype=torch.float32, device="cuda")
    mfa.decode_attention_ex(t["q"], t["k"], t["v"], t["page_table"], t["seq_lens"], out,
                            dec.softmax_scale, num_splits=num_splits, lse_out=lse)
    assert mfa.read_status() == 0
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


def _check_two_calls(dec, num_splits=0):
    t = to_dev(dec)
    want, want_lse = _reference(t, dec, num_splits)
    for _ in range(2):  # the shared array keeps the previous call's contents
        out = torch.full((dec.batch, 64, 256), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((dec.batch, 64), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(t, dec, out, lse, num_splits) == 0
        assert mfa.read_status() == 0
        got = out.double().cpu().numpy()
        assert_close(got, want, decode_atol(dec, want, torch.float32), "noalloc vs ex")
        got_lse = lse.double().cpu().numpy()
        fin = np.isfinite(want_lse)
        assert np.array_equal(np.isneginf(got_lse), np.isneginf(want_lse))
        assert_close(got_lse[fin], want_lse[fin], 1e-4 + 1e-5 * np.abs(want_lse[fin]), "lse")


def test_noalloc_contiguous_matches_workspace_entry_point():
    lens = [4096, 1, 129, 3000, 0, 777, 8192, 64]
    _check_two_calls(gen.make_decode_inputs(401, len(lens), lens))


def test_noalloc_paged_fixed_splits_matches_workspace_entry_point():
    lens = [2000, 65, 5000, 1]
    _check_two_calls(gen.make_decode_inputs(402, len(lens), lens, page_size=64), num_splits=4)


def test_noalloc_allocates_no_device_memory():
    """After a first call (which looks up the array's address), further calls
    change neither the device's free memory nor torch's allocations."""
    lens = [4096, 17, 2000, 0, 5000]
    dec = gen.make_decode_inputs(404, len(lens), lens)
    t = to_dev(dec)
    out = torch.empty(dec.batch, 64, 256, dtype=torch.float32, device="cuda")
    assert _noalloc(t, dec, out) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    alloc0 = torch.cuda.memory_allocated()
    for splits in (0, 3):
        assert _noalloc(t, dec, out, None, splits) == 0
    torch.cuda.synchronize()
    assert mfa.read_status() == 0
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0 and torch.cuda.memory_allocated() == alloc0


def test_noalloc_fp8_through_the_python_wrapper():
    """FP8 cache with per-tensor scales, through mfa.decode_attention_noalloc,
    twice in a row, against mfa.decode_attention_ex (3e-2, the FP8 bound)."""
    lens = [4096, 1, 300, 2500]
    dec = gen.make_decode_inputs(405, len(lens), lens, kv_dtype="e4m3")
    t = to_dev(dec)
    want = torch.empty(dec.batch, 64, 256, dtype=torch.float32, device="cuda")
    mfa.decode_attention_ex(t["q"], t["k"], t["v"], None, t["seq_lens"], want,
                            dec.softmax_scale, "e4m3", k_scale=dec.k_scale, v_scale=dec.v_scale)
    assert mfa.read_status() == 0
    want = want.double().cpu().numpy()
    for _ in range(2):
        got = torch.full((dec.batch, 64, 256), float("nan"), dtype=torch.float32, device="cuda")
        mfa.decode_attention_noalloc(t["q"], t["k"], t["v"], None, t["seq_lens"], got,
                                     dec.softmax_scale, "e4m3", k_scale=dec.k_scale,
                                     v_scale=dec.v_scale)
        assert mfa.read_status() == 0
        got = got.double().cpu().numpy()
        assert_close(got, want, decode_atol(dec, want, torch.float32, base=3e-2), "fp8 noalloc")


def test_noalloc_rejects_requests_beyond_its_array():
    # 400 sequences x 1024 splits needs far more than the fixed 24 MiB array
    dec = gen.make_decode_inputs(403, 400, 1)
    t = to_dev(dec)
    out = torch.empty(400, 64, 256, dtype=torch.float32, device="cuda")
    assert _noalloc(t, dec, out, None, num_splits=1024) == mfa.STATUS_CODES["MFA_ERR_WORKSPACE"]
