"""Parity of mfa_lse_merge (the exchange step of a sequence split across GPUs)
with the oracle, through the C ABI.

Direct cases merge seeded parts (outputs ~ N(0, 1), lse ~ N(0, 4), some parts
empty with NaN outputs) and compare every element with the oracle's float64
merge of the same float32 parts. Tolerance: the kernel merges in fp32 with the
hardware exp2 (relative error ~2^-22 per weight), so |err| <= 1e-5 max|O| for
f32 outputs, plus 2^-8 |ref| (one bf16 rounding) for bf16 outputs; lse to
1e-5 (1 + |lse|).

The split cases emulate the ranks on one GPU as independent calls (no kernel
waits on another): each key range of every sequence is attended by
mfa_decode_attention_ex over its own local cache, and the stacked parts are
merged; the result must match the oracle over the whole sequence within the
decode tolerance (2e-3 on f32 outputs).
"""
import numpy as np
import pytest
import torch

from decode_attention_08_b200 import inputs as gen
from decode_attention_08_b200 import mfa, seqshard
from oracle import oracle as orc

from helpers import assert_close, decode_atol, oracle_decode

pytestmark = pytest.mark.gpu


def _oracle_merge(o_parts, lse_parts):
    S, B, H, D = o_parts.shape
    out = np.zeros((B, H, D))
    lse = np.zeros((B, H))
    for b in range(B):
        for h in range(H):
            w = lse_parts[:, b, h]
            o = np.where(np.isfinite(w)[:, None], o_parts[:, b, h], 0.0)  # empty parts: no weight
            out[b, h], lse[b, h] = orc.combine(o.astype(np.float64), w.astype(np.float64))
    return out, lse


def _run_merge(inp, out_dtype=torch.float32, views=False):
    o = inp.o_parts.cuda()
    l = inp.lse_parts.cuda()
    if views:  # strided views: every part and sequence sits inside a wider buffer
        S, B = o.shape[:2]
        big = torch.full((S + 1, B + 2, 64, 264), float("nan"), device="cuda")
        big[1:, 2:, :, 8:] = o
        o = big[1:, 2:, :, 8:]
        lb = torch.full((S, B, 80), float("nan"), device="cuda")
        lb[:, :, 16:] = l
        l = lb[:, :, 16:]
    B = o.shape[1]
    out = torch.full((B, 64, 256), float("nan"), dtype=out_dtype, device="cuda")
    lse = torch.full((B, 64), float("nan"), device="cuda")
    mfa.lse_merge(o, l, out, lse)
    assert mfa.read_status() == 0
    return out.double().cpu().numpy(), lse.double().cpu().numpy()


@pytest.mark.parametrize("parts,batch,empty", [(1, 3, 0.0), (2, 5, 0.0), (8, 8, 0.2),
                                                (13, 4, 0.5), (64, 2, 0.1)])
def test_merge_matches_oracle_every_element(parts, batch, empty):
    inp = gen.make_lse_merge_inputs(500 + parts, parts, batch, empty=empty)
    got, got_lse = _run_merge(inp)
    ref, ref_lse = _oracle_merge(inp.o_parts.double().numpy(), inp.lse_parts.double().numpy())
    assert_close(got, ref, np.full(ref.shape, 1e-5 * np.nanmax(np.abs(inp.o_parts.numpy()))),
                 "merged output")
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got_lse), fin)
    assert_close(got_lse[fin], ref_lse[fin], 1e-5 * (1 + np.abs(ref_lse[fin])), "merged lse")


def test_merge_bf16_output_and_strided_views():
    inp = gen.make_lse_merge_inputs(77, 6, 5, empty=0.25)
    got, got_lse = _run_merge(inp, torch.bfloat16, views=True)
    ref, ref_lse = _oracle_merge(inp.o_parts.double().numpy(), inp.lse_parts.double().numpy())
    tol = 1e-5 * np.nanmax(np.abs(inp.o_parts.numpy())) + 2.0 ** -8 * np.abs(ref)
    assert_close(got, ref, tol, "merged bf16 output")
    fin = np.isfinite(ref_lse)
    assert_close(got_lse[fin], ref_lse[fin], 1e-5 * (1 + np.abs(ref_lse[fin])), "merged lse")


def test_all_parts_empty_gives_zeros_and_minus_inf():
    inp = gen.make_lse_merge_inputs(5, 4, 3, empty=1.0)
    got, got_lse = _run_merge(inp)
    assert np.array_equal(got, np.zeros_like(got))
    assert np.all(got_lse == -np.inf)


def test_single_part_is_returned_exactly():
    inp = gen.make_lse_merge_inputs(6, 1, 4)
    got, got_lse = _run_merge(inp)
    # weight exp(0) = 1 and 1 / 1 = 1: the one part passes through unchanged
    assert np.array_equal(got, inp.o_parts[0].double().numpy())
    assert np.array_equal(got_lse.astype(np.float32), inp.lse_parts[0].numpy())


def _local_cache(dec, rank, world):
    """Rank `rank`'s local cache: its key range of every sequence (contiguous)."""
    lens = dec.seq_lens.tolist()
    starts, counts = seqshard.local_lengths(lens, rank, world)
    B = len(lens)
    lmax = max([1] + counts)
    k = torch.zeros((B, lmax, 256), dtype=dec.k.dtype)
    v = torch.zeros_like(k)
    for b, (a, n) in enumerate(zip(starts, counts)):
        k[b, :n] = dec.k[b, a:a + n]
        v[b, :n] = dec.v[b, a:a + n]
    return k.cuda(), v.cuda(), torch.tensor(counts, dtype=torch.int32).cuda()


@pytest.mark.parametrize("world,kv_dtype", [(2, "bf16"), (3, "bf16"), (8, "bf16"), (4, "e4m3")])
def test_sequence_split_over_ranks_equals_whole(world, kv_dtype):
    lens = [5000, 129, 1000, 300]   # 129 and 300 leave most ranks an empty range
    dec = gen.make_decode_inputs(600 + world, len(lens), lens, kv_dtype=kv_dtype)
    q = dec.q.cuda()
    o_parts = torch.empty(world, len(lens), 64, 256, device="cuda")
    lse_parts = torch.empty(world, len(lens), 64, device="cuda")
    for r in range(world):   # independent calls, one per emulated rank
        k, v, n = _local_cache(dec, r, world)
        mfa.decode_attention_ex(q, k, v, None, n, o_parts[r], dec.softmax_scale, dec.kv_dtype,
                                k_scale=dec.k_scale, v_scale=dec.v_scale, lse_out=lse_parts[r])
    out = torch.full((len(lens), 64, 256), float("nan"), device="cuda")
    lse = torch.full((len(lens), 64), float("nan"), device="cuda")
    mfa.lse_merge(o_parts, lse_parts, out, lse)
    assert mfa.read_status() == 0
    ref, ref_lse = oracle_decode(dec)
    got = out.double().cpu().numpy()
    got_lse = lse.double().cpu().numpy()
    tol = decode_atol(dec, ref, torch.float32, base=3e-2 if kv_dtype == "e4m3" else 2e-3)
    assert_close(got, ref, tol, f"split over {world}")
    assert_close(got_lse, ref_lse, 1e-4 + 1e-5 * np.abs(ref_lse), "lse")
    # and against the same kernel over the whole sequences
    whole = torch.empty_like(out)
    t = dict(q=q, k=dec.k.cuda(), v=dec.v.cuda(), seq_lens=dec.seq_lens.cuda())
    mfa.decode_attention_ex(t["q"], t["k"], t["v"], None, t["seq_lens"], whole,
                            dec.softmax_scale, dec.kv_dtype, k_scale=dec.k_scale,
                            v_scale=dec.v_scale)
    assert mfa.read_status() == 0
    diff = (whole - out).abs().max().item()
    assert diff <= (3e-2 if kv_dtype == "e4m3" else 2e-3), diff


def test_sharded_decode_through_a_process_group():
    """seqshard.sharded_decode end to end on one GPU: a one-rank NCCL group (the
    all-gather then holds this rank's part only), so the call must equal the
    oracle over the whole sequences."""
    import datetime
    import os
    import socket

    import torch.distributed as dist
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        lens = [1000, 129]
        dec = gen.make_decode_inputs(650, len(lens), lens)
        k, v, n = _local_cache(dec, 0, 1)
        out = torch.full((len(lens), 64, 256), float("nan"), device="cuda")
        lse = torch.full((len(lens), 64), float("nan"), device="cuda")
        seqshard.sharded_decode(dec.q.cuda(), k, v, n, out, softmax_scale=dec.softmax_scale,
                                lse_out=lse)
        assert mfa.read_status() == 0
        ref, ref_lse = oracle_decode(dec)
        got = out.double().cpu().numpy()
        assert_close(got, ref, decode_atol(dec, ref, torch.float32), "sharded")
        assert_close(lse.double().cpu().numpy(), ref_lse,
                     1e-4 + 1e-5 * np.abs(ref_lse), "sharded lse")
    finally:
        dist.destroy_process_group()
