"""Multi-rank host path on CPU: sharding, gathers and timing reductions.

Query rows (and decode sequences) are independent, so N GPUs split a chunk
into row blocks with no exchange in the data path.  These tests check the
row and sequence partitions and run the multi-rank plumbing as two gloo
ranks on the CPU, with the oracle standing in for each rank's indexer call:
the gathered per-rank results must equal one rank's result over the whole
chunk, and the timing reduction must give the slowest rank.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from sparse_attention_token_03_b200.shard import (gather_row_blocks, max_over_ranks, row_shards,
                                                  sequence_shards, shard_pairs, sum_over_ranks)
from synth import make_decode, make_prefill


def _visible(T_q, off, b, e):
    return sum(off + t + 1 for t in range(b, e))


@pytest.mark.parametrize("T_q,off,world", [(1024, 0, 2), (16384, 0, 8), (8192, 122880, 4),
                                           (4096, 1044480, 8), (7, 0, 3), (1, 5, 2), (0, 9, 4),
                                           (3, 0, 8)])
def test_row_shards_cover_and_balance(T_q, off, world):
    blocks = row_shards(T_q, off, world)
    assert len(blocks) == world
    assert blocks[0][0] == 0 and blocks[-1][1] == T_q
    assert all(blocks[r][1] == blocks[r + 1][0] for r in range(world - 1))
    assert all(b <= e for b, e in blocks)
    total = _visible(T_q, off, 0, T_q) if T_q < 20000 else T_q * (off + 1) + T_q * (T_q - 1) // 2
    assert sum(shard_pairs(T_q, off, bl) for bl in blocks) == total
    # each block's work is within one row's work (the heaviest row, off + T_q) of total / world
    for bl in blocks:
        assert abs(shard_pairs(T_q, off, bl) - total / world) <= off + T_q + 1e-9


def test_row_shards_balance_by_pairs_not_rows():
    # a causal chunk from position 0: the first block must hold more rows
    # than the last, since later rows see more keys
    (b0, e0), (b1, e1) = row_shards(16384, 0, 2)
    assert (e0 - b0) > (e1 - b1)
    assert abs((e0 - b0) - 16384 / 2 ** 0.5) < 2  # sqrt(1/2) of the rows hold half the pairs


def test_sequence_shards():
    sl = [10, 10, 10, 10, 1000, 1, 1, 1]
    blocks = sequence_shards(sl, 2)
    assert blocks[0][0] == 0 and blocks[-1][1] == len(sl) and blocks[0][1] == blocks[1][0]
    work = [sum(sl[b:e]) for b, e in blocks]
    assert all(abs(v - sum(sl) / 2) <= max(sl) for v in work)
    assert blocks == [(0, 4), (4, 8)]  # the boundary nearest to half the work
    assert sequence_shards([5] * 8, 4) == [(0, 2), (2, 4), (4, 6), (6, 8)]
    assert sequence_shards([], 2) == [(0, 0), (0, 0)]


def test_single_process_helpers_are_identity():
    assert not dist.is_initialized()
    assert max_over_ranks(2.5) == 2.5 and sum_over_ranks(7) == 7
    t = torch.arange(6).reshape(3, 2)
    assert gather_row_blocks(t, [(0, 3)]) is t


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ["OMP_NUM_THREADS"] = "2"
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # prefill chunk: each rank scores its own row block against all keys
        T_q, off, T_k, topk = 37, 150, 187, 48
        x = make_prefill("causal_1k_h64", T_q=T_q, T_k=T_k, q_offset=off, seed=77)
        blocks = row_shards(T_q, off, world)
        b, e = blocks[rank]
        idx, sc, _ = oracle.prefill_topk(x["q"], x["w"], x["k"], off, topk,
                                         rows=np.arange(b, e, dtype=np.int64), n_threads=2)
        res["p_idx"] = gather_row_blocks(torch.from_numpy(idx), blocks).numpy()
        res["p_score"] = gather_row_blocks(torch.from_numpy(sc), blocks).numpy()
        res["p_pairs"] = sum_over_ranks(shard_pairs(T_q, off, blocks[rank]))
        # decode batch: each rank takes a block of sequences
        y = make_decode("decode_64x128k_h64", B=5, t_cap=90, seed=78)
        sblocks = sequence_shards(y["seq_len"], world)
        sb, se = sblocks[rank]
        if se > sb:
            didx, dsc, _ = oracle.decode_topk(y["q"][sb:se], y["w"][sb:se], y["k"][sb:se],
                                              y["seq_len"][sb:se], 16, n_threads=2)
        else:
            didx, dsc = np.zeros((0, 16), np.int32), np.zeros((0, 16), np.float64)
        res["d_idx"] = gather_row_blocks(torch.from_numpy(didx), sblocks).numpy()
        # a block that is empty on one rank still gathers
        eb = row_shards(1, 4, world)
        mine = torch.full((eb[rank][1] - eb[rank][0], 3), rank + 1, dtype=torch.int32)
        res["empty_gather"] = gather_row_blocks(mine, eb).numpy()
        # slowest rank's time, and the whole-job rate built from it
        res["t_max"] = max_over_ranks(1.5 + 2.0 * rank)
        res["rate"] = res["p_pairs"] / res["t_max"]
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), **res)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_one_rank(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
            p.join()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]

    T_q, off, T_k, topk = 37, 150, 187, 48
    x = make_prefill("causal_1k_h64", T_q=T_q, T_k=T_k, q_offset=off, seed=77)
    idx, sc, _ = oracle.prefill_topk(x["q"], x["w"], x["k"], off, topk)
    y = make_decode("decode_64x128k_h64", B=5, t_cap=90, seed=78)
    didx, _, _ = oracle.decode_topk(y["q"], y["w"], y["k"], y["seq_len"], 16)
    for r in range(world):
        got = np.load(tmp_path / f"rank{r}.npz")
        assert np.array_equal(got["p_idx"], idx)
        assert np.array_equal(got["p_score"], sc)
        assert int(got["p_pairs"]) == _visible(T_q, off, 0, T_q)
        assert np.array_equal(got["d_idx"], didx)
        eb = row_shards(1, 4, world)
        want = np.concatenate([np.full((e - b, 3), i + 1, np.int32) for i, (b, e) in enumerate(eb)])
        assert np.array_equal(got["empty_gather"], want)
        assert float(got["t_max"]) == 1.5 + 2.0 * (world - 1)
        assert float(got["rate"]) == _visible(T_q, off, 0, T_q) / (1.5 + 2.0 * (world - 1))
