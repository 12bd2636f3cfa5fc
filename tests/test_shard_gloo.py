"""Multi-rank host logic of mxfp4_block_scaled_fos_b200.shard on CPU ranks.

Two gloo ranks (spawned processes) each quantize their shard with the
per-shard calls on the oracle.  Rank 0 gathers the pieces and checks that
they equal one unsharded oracle call bit for bit: codes, scales, choice bits
and S_t.  This covers what sharding adds (row ranges on 16-row boundaries,
the amax all-reduce, the global element offset of the SR draws) without a
GPU.  The per-shard CUDA calls themselves are checked against the oracle by
the GPU parity tests.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from mxfp4_block_scaled_fos_b200 import shard, workloads

FMT = {"nvfp4_46": oracle.FMT_NVFP4_46, "nvfp4_6": oracle.FMT_NVFP4_6, "mxfp4": oracle.FMT_MXFP4}
BLK = {"1x16": oracle.BLK_1X16, "16x16": oracle.BLK_16X16, "1x32": oracle.BLK_1X32}
RND = {"rne": oracle.RND_RNE, "sr": oracle.RND_SR}


class OracleOps:
    """The two per-shard calls, on the CPU oracle."""

    @staticmethod
    def amax(x, rht=False, seed=0):
        return torch.from_numpy(oracle.amax(workloads.bits(x), rht=rht, seed=seed).copy())

    @staticmethod
    def quantize(x, amax, elem_offset, fmt="nvfp4_46", block="1x16", rounding="rne", rht=False,
                 seed=0, colwise=False):
        return oracle.quantize(workloads.bits(x), FMT[fmt], BLK[block], RND[rounding], rht, seed,
                               elem_offset, True, colwise,
                               amax.numpy() if amax is not None else None)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bits_of(bitmap, n):
    return np.unpackbits(bitmap, bitorder="little")[:n]


def _input(rows, cols, batch=1):
    g = torch.Generator().manual_seed(11)
    x = torch.randn(batch, rows, cols, generator=g)
    x[..., ::37] *= 30.0
    return x.to(torch.bfloat16)


def _row_worker(rank, world, port, rows, cols, kw, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x = _input(rows, cols)
        lo, hi = shard.row_range(rows, world, rank)
        got = shard.quantize_row_shard(x[:, lo:hi], lo, cols, ops=OracleOps, **kw)
        pieces = [None] * world
        dist.all_gather_object(pieces, (lo, hi, got))
        if rank == 0:
            np.save(out_path, np.array(pieces, dtype=object), allow_pickle=True)
    finally:
        dist.destroy_process_group()


def _entry_worker(rank, world, port, batch, rows, cols, kw, out_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        x = _input(rows, cols, batch)
        lo, hi = shard.batch_range(batch, world, rank)

        def no_collective(*a, **k):
            raise AssertionError("entry sharding must not run a collective")

        real = dist.all_reduce
        dist.all_reduce = no_collective
        try:
            got = shard.quantize_entry_shard(x[lo:hi], lo, rows, cols, ops=OracleOps, **kw)
        finally:
            dist.all_reduce = real
        pieces = [None] * world
        dist.all_gather_object(pieces, (lo, hi, got))
        if rank == 0:
            np.save(out_path, np.array(pieces, dtype=object), allow_pickle=True)
    finally:
        dist.destroy_process_group()


def test_split_range_covers_and_aligns():
    for n in (0, 1, 15, 16, 17, 80, 1000, 4096):
        for world in (1, 2, 3, 4, 8):
            ranges = [shard.row_range(n, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == n
            for (a, b), (c, d) in zip(ranges, ranges[1:]):
                assert b == c
            for a, b in ranges:
                assert a % 16 == 0 and a <= b
            sizes = [b - a for a, b in ranges[:-1]]
            if sizes:
                assert max(sizes) - min(sizes) <= 16
    assert shard.batch_range(128, 8, 7) == (112, 128)
    with pytest.raises(ValueError):
        shard.row_range(16, 2, 2)


@pytest.mark.parametrize("kw", [
    dict(fmt="nvfp4_46", rounding="sr", colwise=True, seed=5),
    dict(fmt="nvfp4_46", rht=True, seed=3),
    dict(fmt="nvfp4_46", block="16x16", colwise=True),
    dict(fmt="nvfp4_6"),
], ids=["sr_dual", "rht", "2d", "six_only"])
def test_row_shards_equal_one_call(tmp_path, kw):
    rows, cols, world = 80, 64, 2     # 5 row tiles: a 3 + 2 split
    out = str(tmp_path / "pieces.npy")
    mp.spawn(_row_worker, args=(world, _free_port(), rows, cols, kw, out), nprocs=world, join=True)
    pieces = np.load(out, allow_pickle=True)
    full = OracleOps.quantize(_input(rows, cols), None, 0, **kw)
    block = kw.get("block", "1x16")
    np.testing.assert_array_equal(np.concatenate([p[2]["r_codes"] for p in pieces], axis=1),
                                  full["r_codes"])
    np.testing.assert_array_equal(np.concatenate([p[2]["r_scales"] for p in pieces], axis=1),
                                  full["r_scales"])
    for p in pieces:
        np.testing.assert_array_equal(p[2]["tensor_scale"], full["tensor_scale"])
    if block == "16x16":
        per_row_tile = cols // 16
        bits = [_bits_of(p[2]["r_choice"], (p[1] - p[0]) // 16 * per_row_tile) for p in pieces]
        np.testing.assert_array_equal(np.concatenate(bits),
                                      _bits_of(full["r_choice"], rows // 16 * per_row_tile))
    else:
        bits = [_bits_of(p[2]["r_choice"], (p[1] - p[0]) * cols // 16) for p in pieces]
        np.testing.assert_array_equal(np.concatenate(bits), _bits_of(full["r_choice"], rows * cols // 16))
    if kw.get("colwise"):
        np.testing.assert_array_equal(np.concatenate([p[2]["c_codes"] for p in pieces], axis=2),
                                      full["c_codes"])
        np.testing.assert_array_equal(np.concatenate([p[2]["c_scales"] for p in pieces], axis=2),
                                      full["c_scales"])
        if block != "16x16":
            bits = [_bits_of(p[2]["c_choice"], cols * (p[1] - p[0]) // 16).reshape(cols, -1)
                    for p in pieces]
            np.testing.assert_array_equal(np.concatenate(bits, axis=1).ravel(),
                                          _bits_of(full["c_choice"], cols * rows // 16))


def test_entry_shards_equal_one_call_without_collective(tmp_path):
    batch, rows, cols, world = 3, 32, 48, 2
    kw = dict(fmt="nvfp4_46", rounding="sr", seed=9)
    out = str(tmp_path / "pieces.npy")
    mp.spawn(_entry_worker, args=(world, _free_port(), batch, rows, cols, kw, out), nprocs=world,
             join=True)
    pieces = np.load(out, allow_pickle=True)
    full = OracleOps.quantize(_input(rows, cols, batch), None, 0, **kw)
    for key in ("r_codes", "r_scales", "tensor_scale"):
        np.testing.assert_array_equal(np.concatenate([p[2][key] for p in pieces], axis=0), full[key])
    bits = [_bits_of(p[2]["r_choice"], (p[1] - p[0]) * rows * cols // 16) for p in pieces]
    np.testing.assert_array_equal(np.concatenate(bits), _bits_of(full["r_choice"], batch * rows * cols // 16))
