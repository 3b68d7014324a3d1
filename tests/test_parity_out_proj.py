"""GPU parity of the output projection (``mfa_output_proj``) against the
float64 oracle, through the C ABI.

Tolerance: one bf16 rounding of the result (2^-8 |ref|) plus fp32 accumulation
over K terms (1e-4 max|ref|, as for the query projection).
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa
from oracle import oracle as orc

pytestmark = pytest.mark.gpu


def _run(inp):
    o, w = inp.o.cuda(), inp.w_o.cuda()
    y = torch.full((o.shape[0], w.shape[1]), float("nan"), dtype=torch.bfloat16, device="cuda")
    mfa.output_proj(o, w, y)
    assert mfa.read_status() == 0
    return y.float().cpu().numpy().astype(np.float64)


def _tol(ref):
    return 2.0 ** -8 * np.abs(ref) + 1e-4 * np.abs(ref).max()


@pytest.mark.parametrize("batch,k,n", [(1, 256, 128), (5, 512, 384), (33, 1024, 256)])
def test_small_shapes_all_outputs(batch, k, n):
    g = torch.Generator().manual_seed(800 + batch)
    inp = gen.OutProjInputs(o=torch.randn(batch, k, generator=g).to(torch.bfloat16),
                            w_o=(torch.randn(k, n, generator=g) * 0.05).to(torch.bfloat16))
    got = _run(inp)
    ref = orc.out_proj(gen.bits(inp.o), gen.bits(inp.w_o))
    assert np.all(np.abs(got - ref) <= _tol(ref)), np.abs(got - ref).max()


@pytest.mark.parametrize("batch", [8, 64])
def test_step3_shape(batch):
    """[B, 16384] x [16384, 7168], compared on every output (float64 oracle, OpenMP)."""
    inp = gen.make_out_proj_inputs(810 + batch, batch)
    got = _run(inp)
    ref = orc.out_proj(gen.bits(inp.o), gen.bits(inp.w_o))
    assert np.all(np.abs(got - ref) <= _tol(ref)), np.abs(got - ref).max()
