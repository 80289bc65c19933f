"""Row-sharded products (decode_packed_bit_b200/shard.py) on the CPU: the
shard bounds for ragged N, and two gloo ranks that each multiply their rows
of every matrix and all-gather, reassembled and compared with the one-rank
result of the oracle.  The local product on each rank is the oracle (no GPU
here); on GPUs it is the library's group call."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from decode_packed_bit_b200.shard import ShardLayout, assemble, row_shard, shard_sizes  # noqa: E402


@pytest.mark.parametrize("N", [0, 1, 31, 32, 33, 300, 4096, 5120, 11008, 17408, 17409])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_row_shard_covers_rows_once(N, world):
    prev = 0
    sizes = []
    for q in range(world):
        n0, n1 = row_shard(N, world, q)
        assert n0 == prev and n1 >= n0          # contiguous, in rank order
        assert n0 % 32 == 0 or n0 == N          # starts on a 32-row tile
        prev = n1
        sizes.append(n1 - n0)
    assert prev == N                            # every row exactly once
    tiles = [-(-s // 32) for s in sizes]
    assert max(tiles) - min(tiles) <= 1         # balanced to one tile
    assert sizes == shard_sizes(N, world)


def test_row_shard_rejects_bad_arguments():
    with pytest.raises(ValueError):
        row_shard(10, 0, 0)
    with pytest.raises(ValueError):
        row_shard(10, 2, 2)


def test_assemble_places_every_rank_segment():
    lay = ShardLayout(R=3, M=2, N=70, world=3)   # shards 32, 32, 6 rows
    buf = np.full(lay.world * lay.segment, np.nan, np.float32)
    ref = np.arange(3 * 2 * 70, dtype=np.float32).reshape(3, 2, 70)
    for q in range(3):
        n0, n1 = lay.bounds(q)
        for r in range(3):
            base = q * lay.segment + r * lay.slot
            buf[base:base + 2 * (n1 - n0)] = ref[r, :, n0:n1].ravel()
    assert np.array_equal(assemble(buf, lay), ref)
    assert lay.slot % 4 == 0


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(fmt, R, M, N, K):
    import oracle
    import synth
    mats = []
    for r in range(R):
        if fmt == "q1":
            bits = oracle.pack("q1", synth.q1_codes(500 + r, N, K))
            sc = synth.q1_scales(500 + r, N, K)
        else:
            bits = oracle.pack("int4", synth.int4_codes(500 + r, N, K))
            sc = synth.int4_scales(500 + r, N, K)
        mats.append((bits, sc))
    x = synth.bf16_normal(599, (M, K))
    return mats, x


def _rank_main(rank, world, port, out_dir, fmt, R, M, N, K):
    sys.path.insert(0, ROOT)
    import oracle
    from decode_packed_bit_b200.shard import RowShardedGroup, row_shard
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        mats, x = _problem(fmt, R, M, N, K)
        n0, n1 = row_shard(N, world, rank)
        bits = [torch.from_numpy(b[n0:n1].copy()) for b, _ in mats]
        scales = [torch.from_numpy(s[n0:n1].copy().view(np.int16)) for _, s in mats]
        prod = oracle.q1_gemv if fmt == "q1" else oracle.int4_gemv

        def local_product(bs, ss, xx, ys):   # this rank's rows, on the host
            for b, s, y in zip(bs, ss, ys):
                y.copy_(torch.from_numpy(prod(b.numpy(), s.numpy().view(np.uint16), xx).astype(np.float32)))

        grp = RowShardedGroup(fmt, bits, scales, N, K, M, local_product=local_product)
        grp.step(x)
        np.save(os.path.join(out_dir, f"y{rank}.npy"), grp.dense().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fmt,R,M,N,K", [("q1", 3, 1, 300, 256), ("q1", 2, 4, 70, 128), ("int4", 2, 2, 96, 128)])
def test_two_gloo_ranks_reassemble_the_one_rank_result(tmp_path, fmt, R, M, N, K):
    import oracle
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), fmt, R, M, N, K), nprocs=world,
                       start_method="spawn")
    mats, x = _problem(fmt, R, M, N, K)
    prod = oracle.q1_gemv if fmt == "q1" else oracle.int4_gemv
    ref = np.stack([prod(b, s, x) for b, s in mats]).astype(np.float32)
    for rank in range(world):
        got = np.load(tmp_path / f"y{rank}.npy")
        assert got.shape == (R, M, N)
        assert np.array_equal(got, ref)   # every rank holds all of y, in the one-rank order
