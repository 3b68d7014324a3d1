"""GPU tests of the decode workspace's hand-off between the call's two kernels.

The combine kernel starts while the attention kernel still runs and merges a
split sequence once the flags of all its partial slots are set. Every word it
reads (the per-sequence plan words, the per-slot flags) is written by the
attention kernel of the same call before the combine kernel may start, so a
workspace needs no initialisation and nothing left in it by an earlier call,
of any shape, or by anything else, can change a result.

Each test compares against a call on a fresh workspace, which the parity tests
tie to the oracle; results must be bit-identical, because the split plan (and
so the arithmetic) does not depend on the workspace.
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa

from helpers import run_decode, to_dev

pytestmark = pytest.mark.gpu


def _call(t, dec, out, ws, num_splits=0, stream=None):
    mfa.decode_attention_ex(t["q"], t["k"], t["v"], t["page_table"], t["seq_lens"], out,
                            dec.softmax_scale, dec.kv_dtype, k_scale=dec.k_scale,
                            v_scale=dec.v_scale, num_splits=num_splits, workspace=ws,
                            stream=stream)


def _fresh(dec, num_splits=0):
    return run_decode(dec, num_splits=num_splits)


def _mixed(seed, batch, lmax):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, lmax + 1, size=batch).tolist()
    lens[0] = lmax  # one long sequence: split across many CTAs
    return gen.make_decode_inputs(seed, batch, lens, lmax=lmax)


def _garbage(ws, kind, seed=0):
    """Fill a workspace with a pattern a caller's memory might hold."""
    if kind == "random":
        g = torch.Generator(device="cuda").manual_seed(seed)
        ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device="cuda", generator=g))
    elif kind == "ones":
        ws.fill_(0xFF)
    elif kind == "small_ints":  # words of 1: every flag "set"
        ws.view(torch.int32).fill_(1)
    else:
        ws.zero_()


@pytest.mark.parametrize("kind", ["random", "ones", "small_ints"])
@pytest.mark.parametrize("num_splits", [0, 5])
def test_garbage_filled_workspace(kind, num_splits):
    dec = _mixed(601, 40, 6000)
    want = _fresh(dec, num_splits)
    t = to_dev(dec)
    ws = torch.empty(mfa.decode_workspace_size(dec.batch, num_splits), dtype=torch.uint8,
                     device="cuda")
    for i in range(2):
        _garbage(ws, kind, seed=i)
        out = torch.full((dec.batch, 64, 256), float("nan"), dtype=torch.float32, device="cuda")
        _call(t, dec, out, ws, num_splits)
        assert mfa.read_status() == 0
        assert np.array_equal(out.double().cpu().numpy(), want), (kind, i)


def test_workspace_freed_and_reallocated_at_the_same_address():
    """A caching allocator hands a freed block back at the same address with
    whatever it last held: here the words another call (another batch size)
    left, then random bytes. No memset in between."""
    a = _mixed(602, 64, 5000)
    b = _mixed(603, 5, 9000)
    want_a, want_b = _fresh(a), _fresh(b)
    ta, tb = to_dev(a), to_dev(b)
    need = max(mfa.decode_workspace_size(64, 0), mfa.decode_workspace_size(5, 0))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    addr = ws.data_ptr()
    out_a = torch.empty(64, 64, 256, dtype=torch.float32, device="cuda")
    _call(ta, a, out_a, ws)
    assert mfa.read_status() == 0
    del ws
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")  # same block, contents kept
    out_b = torch.full((5, 64, 256), float("nan"), dtype=torch.float32, device="cuda")
    _call(tb, b, out_b, ws)
    assert mfa.read_status() == 0
    assert np.array_equal(out_b.double().cpu().numpy(), want_b)
    del ws
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    _garbage(ws, "random", seed=7)
    out_a.fill_(float("nan"))
    _call(ta, a, out_a, ws)
    assert mfa.read_status() == 0
    assert np.array_equal(out_a.double().cpu().numpy(), want_a)
    print("same address reused:", ws.data_ptr() == addr)


def test_one_workspace_across_batch_sizes_and_split_modes():
    big = _mixed(602, 64, 5000)
    small = _mixed(603, 5, 9000)
    paged = gen.make_decode_inputs(604, 3, [3000, 1, 700], page_size=32)
    want = {
        ("big", 0): _fresh(big),
        ("small", 0): _fresh(small),
        ("small", 3): _fresh(small, 3),
        ("paged", 0): _fresh(paged),
    }
    need = max(mfa.decode_workspace_size(d.batch, s)
               for d, s in ((big, 0), (small, 0), (small, 3), (paged, 0)))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    _garbage(ws, "random", seed=3)
    tens = {"big": (big, to_dev(big)), "small": (small, to_dev(small)),
            "paged": (paged, to_dev(paged))}
    order = [("big", 0), ("small", 0), ("big", 0), ("small", 3), ("paged", 0), ("small", 0),
             ("big", 0), ("big", 0)]
    for name, splits in order:
        dec, t = tens[name]
        out = torch.full((dec.batch, 64, 256), float("nan"), dtype=torch.float32, device="cuda")
        _call(t, dec, out, ws, num_splits=splits)
        assert mfa.read_status() == 0
        got = out.double().cpu().numpy()
        assert np.array_equal(got, want[(name, splits)]), (name, splits)


def test_back_to_back_calls_without_host_sync():
    a = _mixed(605, 32, 7000)
    b = _mixed(606, 32, 3000)
    want_a, want_b = _fresh(a), _fresh(b)
    ta, tb = to_dev(a), to_dev(b)
    ws = torch.empty(mfa.decode_workspace_size(32, 0), dtype=torch.uint8, device="cuda")
    outs = [torch.empty(32, 64, 256, dtype=torch.float32, device="cuda") for _ in range(12)]
    for i, out in enumerate(outs):
        dec, t = (a, ta) if i % 2 == 0 else (b, tb)
        _call(t, dec, out, ws)
    assert mfa.read_status() == 0
    for i, out in enumerate(outs):
        want = want_a if i % 2 == 0 else want_b
        assert np.array_equal(out.double().cpu().numpy(), want), i


@pytest.mark.parametrize("calls_per_graph", [1, 3])
def test_graph_replays(calls_per_graph):
    dec = _mixed(607, 48, 6000)
    t = to_dev(dec)
    ws = torch.empty(mfa.decode_workspace_size(dec.batch, 0), dtype=torch.uint8, device="cuda")
    _garbage(ws, "ones")
    out = torch.empty(dec.batch, 64, 256, dtype=torch.float32, device="cuda")
    st = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=st):
        for _ in range(calls_per_graph):
            _call(t, dec, out, ws, stream=st)
    torch.cuda.synchronize()
    qs = [torch.randn_like(t["q"], dtype=torch.float32).to(torch.bfloat16) for _ in range(3)]
    for qi in qs:
        t["q"].copy_(qi)
        g.replay()
        torch.cuda.synchronize()
        assert mfa.read_status() == 0
        dec_i = gen.DecodeInputs(q=qi.cpu(), k=dec.k, v=dec.v, seq_lens=dec.seq_lens)
        assert np.array_equal(out.double().cpu().numpy(), _fresh(dec_i))
    del g
