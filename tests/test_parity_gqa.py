"""GPU parity of the grouped-query (GQA) comparison kernel against the float64
oracle, through the C ABI (mfa_gqa_decode_attention). 64 query heads of
dimension 128 in 2 groups, each with its own 128-wide key and value head (the
same 1024 cache bytes per token as MFA). Every output is compared; the bound is
2e-3 on fp32 outputs (plus one bf16 rounding for bf16 outputs), as for MFA."""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa
from oracle import oracle as orc

from helpers import assert_close

pytestmark = pytest.mark.gpu

RAGGED = [1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 300, 513, 4000]


def _tol(ref, out_dtype):
    tol = np.full(ref.shape, 2e-3)
    if out_dtype == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(ref)
    return tol


def _run(inp, out_dtype=torch.float32, num_splits=0, lse=False):
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    lens = inp.seq_lens.cuda()
    pt = None if inp.page_table is None else inp.page_table.cuda()
    out = torch.full((inp.batch, 64, 128), float("nan"), dtype=out_dtype, device="cuda")
    lse_out = torch.full((inp.batch, 64), float("nan"), device="cuda") if lse else None
    mfa.gqa_decode_attention(q, k, v, pt, lens, out, inp.softmax_scale, num_splits=num_splits,
                             lse_out=lse_out)
    assert mfa.read_status() == 0
    got = out.double().cpu().numpy()
    return (got, lse_out.double().cpu().numpy()) if lse else got


def _oracle(inp):
    pt = None if inp.page_table is None else inp.page_table.numpy()
    return orc.gqa_decode(gen.bits(inp.q), gen.bits(inp.k), gen.bits(inp.v),
                          inp.seq_lens.numpy(), inp.softmax_scale, page_table=pt,
                          page_size=inp.page_size or 64)


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_gqa_ragged_all_outputs(out_dtype):
    inp = gen.make_gqa_inputs(801, len(RAGGED), RAGGED, lmax=4100)
    got, lse = _run(inp, out_dtype, lse=True)
    ref, lref = _oracle(inp)
    err = assert_close(got, ref, _tol(ref, out_dtype), "gqa out")
    assert_close(lse, lref, 1e-4 + 1e-5 * np.abs(lref), "gqa lse")
    print(f"gqa ragged ({out_dtype}): max |err| {err:.2e}")


def test_gqa_single_token_is_its_groups_value_row():
    inp = gen.make_gqa_inputs(802, 3, [1, 1, 1])
    got = _run(inp)
    for h in range(64):
        assert np.array_equal(got[:, h], inp.v[:, 0, h // 32].double().numpy())


def test_gqa_empty_sequences():
    inp = gen.make_gqa_inputs(803, 4, [0, 700, 0, 1])
    got, lse = _run(inp, lse=True)
    assert np.all(got[0] == 0) and np.all(got[2] == 0)
    assert np.all(np.isneginf(lse[0])) and np.all(np.isneginf(lse[2]))
    ref, _ = _oracle(inp)
    assert_close(got, ref, _tol(ref, torch.float32), "gqa empty")


@pytest.mark.parametrize("num_splits", [2, 7])
def test_gqa_fixed_splits(num_splits):
    inp = gen.make_gqa_inputs(804, 4, [5000, 129, 1, 2048])
    got = _run(inp, num_splits=num_splits)
    ref, _ = _oracle(inp)
    assert_close(got, ref, _tol(ref, torch.float32), f"gqa splits={num_splits}")


@pytest.mark.parametrize("page_size", [16, 64, 256])
def test_gqa_paged_is_bit_exact_with_contiguous(page_size):
    lens = [1, 64, 65, 200, 1000, 4097]
    inp = gen.make_gqa_inputs(805 + page_size, len(lens), lens, page_size=page_size)
    L = max(lens)
    kc = torch.zeros(len(lens), L, 2, 128, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    for b, n in enumerate(lens):
        t = torch.arange(n)
        pages = inp.page_table[b, t // page_size].long()
        kc[b, :n] = inp.k[pages, t % page_size]
        vc[b, :n] = inp.v[pages, t % page_size]
    cont = gen.GqaInputs(q=inp.q, k=kc, v=vc, seq_lens=inp.seq_lens)
    got_p, lse_p = _run(inp, lse=True)
    got_c, lse_c = _run(cont, lse=True)
    assert np.array_equal(got_p, got_c) and np.array_equal(lse_p, lse_c)
    ref, _ = _oracle(inp)
    assert_close(got_p, ref, _tol(ref, torch.float32), "gqa paged")


def test_gqa_workload_all_outputs():
    inp = gen.make_gqa_workload()
    got = _run(inp)
    assert np.all(np.isfinite(got))
    ref, _ = _oracle(inp)
    err = assert_close(got, ref, _tol(ref, torch.float32), inp.meta["name"])
    print(f"{inp.meta['name']}: max |err| {err:.2e} over {got.size} outputs")


def test_gqa_rejects_other_shapes():
    inp = gen.make_gqa_inputs(806, 2, [10, 20])
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    lens = inp.seq_lens.cuda()
    out = torch.empty(2, 64, 128, device="cuda")
    with pytest.raises(mfa.MfaError):   # three groups
        mfa.gqa_decode_attention(q, torch.cat([k, k[:, :, :1]], 2), torch.cat([v, v[:, :, :1]], 2),
                                 None, lens, out)
    with pytest.raises(mfa.MfaError):   # MFA-shaped q
        mfa.gqa_decode_attention(torch.zeros(2, 64, 256, dtype=torch.bfloat16, device="cuda"),
                                 k, v, None, lens, out)
