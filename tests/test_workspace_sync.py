"""GPU tests of the decode workspace's synchronisation words.

The combine kernel starts while the attention kernel still runs and merges a
split sequence once the last writer of its partials has arrived. The words
that carry this (an arrival counter and four ready words per sequence) sit at
the start of the caller's workspace; every call returns them to zero, and the
library clears them when a workspace is new to it or serves another batch size.

Each test compares against a call on a fresh zero-filled workspace, which the
parity tests tie to the oracle; results must be bit-identical, because the
split plan (and so the arithmetic) does not depend on the workspace.
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


def _sync_words(ws, batch):
    """Arrival counters [B] (u32) and ready words [B][4] (u64) of a workspace."""
    raw = ws.cpu().numpy()
    arrive = raw[:4 * batch].view(np.uint32)
    ready_off = (4 * batch + 15) & ~15
    ready = raw[ready_off:ready_off + 32 * batch].view(np.uint64)
    return arrive, ready


def _mixed(seed, batch, lmax):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, lmax + 1, size=batch).tolist()
    lens[0] = lmax  # one long sequence: split across many CTAs
    return gen.make_decode_inputs(seed, batch, lens, lmax=lmax)


def test_sync_words_are_zero_after_each_call():
    dec = _mixed(601, 40, 6000)
    t = to_dev(dec)
    ws = torch.zeros(mfa.decode_workspace_size(dec.batch, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty(dec.batch, 64, 256, dtype=torch.float32, device="cuda")
    for _ in range(3):
        _call(t, dec, out, ws)
        assert mfa.read_status() == 0
        arrive, ready = _sync_words(ws, dec.batch)
        assert not arrive.any() and not ready.any()


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
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
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
    ws = torch.zeros(mfa.decode_workspace_size(32, 0), dtype=torch.uint8, device="cuda")
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
    ws = torch.zeros(mfa.decode_workspace_size(dec.batch, 0), dtype=torch.uint8, device="cuda")
    out = torch.empty(dec.batch, 64, 256, dtype=torch.float32, device="cuda")
    st = torch.cuda.Stream()
    with torch.cuda.stream(st):
        _call(t, dec, out, ws, stream=st)  # first sight of the workspace: outside capture
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
