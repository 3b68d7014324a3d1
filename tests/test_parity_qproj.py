"""GPU parity of the MFA low-rank query projection q = (x W_qa) W_qb against the
float64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa
from oracle import oracle as orc

from helpers import assert_close

pytestmark = pytest.mark.gpu


def _run(p: gen.ProjInputs, ex=False):
    x, wa, wb = p.x.cuda(), p.w_qa.cuda(), p.w_qb.cuda()
    q = torch.full((x.shape[0], wb.shape[1]), float("nan"), dtype=torch.bfloat16, device="cuda")
    if ex:
        ws = torch.zeros(mfa.query_proj_workspace_size(x.shape[0], x.shape[1], wa.shape[1]),
                         dtype=torch.uint8, device="cuda")
        mfa.query_proj_ex(x, wa, wb, q, ws)
    else:
        mfa.query_proj(x, wa, wb, q)
    assert mfa.read_status() == 0
    return q.double().cpu().numpy()


def _ref(p):
    return orc.query_proj(gen.bits(p.x), gen.bits(p.w_qa), gen.bits(p.w_qb))


def _tol(ref):
    return 2.0 ** -8 * np.abs(ref) + 1e-4 * np.max(np.abs(ref))


@pytest.mark.parametrize("batch", [1, 3, 8, 16, 37, 128])
def test_small_shapes(batch):
    p = gen.make_proj_inputs(300 + batch, batch, hidden=512, rank=256, out_features=384)
    got = _run(p)
    ref = _ref(p)
    assert_close(got, ref, _tol(ref), f"batch={batch}")


def test_ex_with_caller_workspace_twice():
    p = gen.make_proj_inputs(340, 5, hidden=1024, rank=512, out_features=256)
    a = _run(p, ex=True)
    b = _run(p, ex=True)
    assert np.array_equal(a, b)
    ref = _ref(p)
    assert_close(a, ref, _tol(ref), "ex")


def test_step3_shape_batch8():
    """The Step-3 shapes: 7168 -> 2048 -> 64 x 256, batch 8."""
    p = gen.make_proj_inputs(2005, 8)
    got = _run(p)
    ref = _ref(p)
    assert_close(got, ref, _tol(ref), "step3")


@pytest.mark.parametrize("batch", [16, 64])
def test_step3_shape_two_launch_path(batch):
    """Batches above 8 take the two-launch path (split-K latent GEMM, then the
    up-projection); checked at the Step-3 shapes on every output."""
    p = gen.make_proj_inputs(2100 + batch, batch)
    got = _run(p)
    ref = _ref(p)
    assert_close(got, ref, _tol(ref), f"step3 batch {batch}")
