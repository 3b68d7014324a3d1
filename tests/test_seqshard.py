"""Host logic of a sequence split across ranks (CPU, gloo): the key ranges and
the all-gather of the (O, lse) parts.

Each gloo rank stands in for one GPU: it attends over its own key range with
the oracle (the test's stand-in for the rank's decode-attention call), the
package's ``gather_parts`` exchanges the parts, and the oracle's log-sum-exp
merge of the gathered parts must equal the oracle over the whole sequence.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from decode_attention_08_b200 import seqshard


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_key_ranges_are_disjoint_tile_aligned_and_cover(world):
    for L in [0, 1, 127, 128, 129, 300, 1000, 4096, 65536, 65537]:
        ranges = [seqshard.key_range(L, r, world) for r in range(world)]
        pos = 0
        for a, e in ranges:
            assert a == pos and e >= a            # contiguous, in rank order
            assert a % 128 == 0 or a == L          # cut at tile boundaries
            pos = e
        assert pos == L                            # covering
        tiles = [-(-(e - a) // 128) for a, e in ranges]
        assert max(tiles) - min(tiles) <= 1        # balanced to one tile
        assert sum(tiles) == -(-L // 128)


def test_key_range_rejects_bad_arguments():
    for args in [(10, 2, 2), (10, -1, 2), (10, 0, 0), (-1, 0, 1)]:
        with pytest.raises(ValueError):
            seqshard.key_range(*args)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    from decode_attention_08_b200 import inputs as gen
    from decode_attention_08_b200 import seqshard as ss
    from oracle import oracle as orc
    try:
        lens = [300, 100, 1000]   # the 100-token sequence leaves the last rank an empty range
        dec = gen.make_decode_inputs(31, len(lens), lens)
        q, k, v = gen.bits(dec.q), gen.bits(dec.k), gen.bits(dec.v)
        starts, counts = ss.local_lengths(lens, rank, world)
        # this rank's local cache: its key range of every sequence
        lmax = max([1] + counts)
        kl = np.zeros((len(lens), lmax, 256), np.uint16)
        vl = np.zeros_like(kl)
        for b, (a, n) in enumerate(zip(starts, counts)):
            kl[b, :n] = k[b, a:a + n]
            vl[b, :n] = v[b, a:a + n]
        o_loc, lse_loc = orc.decode(q, kl, vl, np.array(counts, np.int32), 1 / 16)
        o_part = torch.from_numpy(o_loc.astype(np.float32))
        lse_part = torch.from_numpy(lse_loc.astype(np.float32))
        o_parts, lse_parts = ss.gather_parts(o_part, lse_part)
        out[rank] = (o_part.numpy(), lse_part.numpy(), o_parts.numpy(), lse_parts.numpy(), counts)
    finally:
        torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_gather_parts_in_rank_order_and_merge_to_the_whole(world):
    from decode_attention_08_b200 import inputs as gen
    from oracle import oracle as orc
    out = mp.Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    lens = [300, 100, 1000]
    assert out[world - 1][4][1] == 0               # the empty range is exercised
    for r in range(world):
        o_parts, lse_parts = out[r][2], out[r][3]
        assert o_parts.shape == (world, 3, 64, 256) and lse_parts.shape == (world, 3, 64)
        for s in range(world):                     # part s is rank s's own part
            np.testing.assert_array_equal(o_parts[s], out[s][0])
            np.testing.assert_array_equal(lse_parts[s], out[s][1])
    dec = gen.make_decode_inputs(31, len(lens), lens)
    full, lse_full = orc.decode(gen.bits(dec.q), gen.bits(dec.k), gen.bits(dec.v),
                                np.array(lens, np.int32), 1 / 16)
    o_parts, lse_parts = out[0][2], out[0][3]
    for b in range(3):
        for h in (0, 9, 63):
            merged, lse = orc.combine(o_parts[:, b, h].astype(np.float64),
                                      lse_parts[:, b, h].astype(np.float64))
            # the parts were rounded to float32 for the exchange
            np.testing.assert_allclose(merged, full[b, h], rtol=1e-5, atol=1e-6)
            assert abs(lse - lse_full[b, h]) < 1e-5 * max(1.0, abs(lse_full[b, h]))
