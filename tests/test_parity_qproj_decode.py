"""GPU parity of mfa_qproj_decode_attention: the query projection followed by
decode attention on its result in one call (the Step-3 decode step's query
path: the 2048-wide bottleneck, then attention over the shared key/value
heads), through the C ABI.

Each call is checked three ways: q against the float64 projection oracle (as
the projection's own tests), the attention output against the float64
attention oracle run on that q (the bf16 query the attention consumed), and
both bit for bit against the two separate calls.
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa
from oracle import oracle as orc

from helpers import assert_close, decode_atol, oracle_decode

pytestmark = pytest.mark.gpu


def _fused_and_separate(dec, proj, num_splits):
    B = dec.batch
    x, wa, wb = proj.x.cuda(), proj.w_qa.cuda(), proj.w_qb.cuda()
    k, v, lens = dec.k.cuda(), dec.v.cuda(), dec.seq_lens.cuda()
    q1 = torch.full((B, 64 * 256), float("nan"), dtype=torch.bfloat16, device="cuda")
    out1 = torch.full((B, 64, 256), float("nan"), dtype=torch.float32, device="cuda")
    lse1 = torch.full((B, 64), float("nan"), device="cuda")
    mfa.qproj_decode_attention(x, wa, wb, q1, k, v, None, lens, out1, dec.softmax_scale,
                               num_splits=num_splits, lse_out=lse1)
    assert mfa.read_status() == 0
    q2 = torch.empty_like(q1)
    out2 = torch.empty_like(out1)
    lse2 = torch.empty_like(lse1)
    mfa.query_proj(x, wa, wb, q2)
    mfa.decode_attention_ex(q2.view(B, 64, 256), k, v, None, lens, out2, dec.softmax_scale,
                            num_splits=num_splits, lse_out=lse2)
    assert mfa.read_status() == 0
    assert torch.equal(q1, q2) and torch.equal(out1, out2) and torch.equal(lse1, lse2)
    return q1.cpu(), out1.double().cpu().numpy()


def _check(dec, proj, num_splits):
    q, got = _fused_and_separate(dec, proj, num_splits)
    qref = orc.query_proj(gen.bits(proj.x), gen.bits(proj.w_qa), gen.bits(proj.w_qb))
    assert_close(q.double().numpy(), qref, 2.0 ** -8 * np.abs(qref) + 1e-4 * np.max(np.abs(qref)),
                 "q")
    dec.q = q.view(dec.batch, 64, 256)   # the query the attention consumed
    ref, _ = oracle_decode(dec)
    return assert_close(got, ref, decode_atol(dec, ref, torch.float32), "out")


@pytest.mark.parametrize("num_splits", [0, 3])
def test_small_projection_then_attention(num_splits):
    lens = [700, 1, 129, 3000]
    dec = gen.make_decode_inputs(901, len(lens), lens)
    proj = gen.make_proj_inputs(902, len(lens), hidden=512, rank=256)
    _check(dec, proj, num_splits)


def test_workload5_fused_call():
    """Batch 8, context 65536, 16-way split, preceded by the Step-3 projection."""
    dec, proj = gen.make_workload(5)
    err = _check(dec, proj, 16)
    print(f"workload 5 fused: max |err| {err:.2e}")
