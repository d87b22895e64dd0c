"""Parity of the fused dense path (prefill and decode) with the fp64 oracle.

Every test calls the C ABI through the Python binding on the GPU and
compares with the oracle on identical seeded inputs (tests/parity.py gives
the tolerance and the tie rule).
"""

import numpy as np
import pytest
import torch

import sparse_attention_token_03_b200 as dsa
from synth import WORKLOADS, make_decode, make_integer_prefill, make_prefill
from tests.parity import check_rows, oracle_decode_rows, oracle_prefill_rows

pytestmark = pytest.mark.gpu


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def run_prefill(x, topk, rows=None):
    idx, sc = dsa.dsa_index_prefill(bf16(x["q"]), f32(x["w"]), bf16(x["k"]), x["q_offset"], topk)
    torch.cuda.synchronize()
    idx, sc = idx.cpu().numpy(), sc.cpu().numpy()
    if rows is not None:
        idx, sc = idx[rows], sc[rows]
    return idx, sc


def check_prefill(x, topk, rows=None, label=""):
    T_q = x["q"].shape[0]
    rows = np.arange(T_q) if rows is None else np.asarray(rows)
    gi, gs = run_prefill(x, topk, rows)
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, topk)
    visible = x["q_offset"] + rows + 1
    return check_rows(gi, gs, oi, osc, amax, visible, topk, score_of, label)


@pytest.mark.parametrize("H", [64, 32])
def test_prefill_tiny_full_causal(H):
    # the oracle-sized causal prefill, every row
    wl = "causal_1k_h64"
    x = make_prefill(wl) if H == 64 else make_prefill("chunk_128k_h32", T_q=1024, T_k=1024, q_offset=0)
    check_prefill(x, 256, label=f"causal1k H{H}")


@pytest.mark.parametrize("T,off,topk", [(1, 0, 1), (37, 0, 5), (777, 0, 100), (300, 123, 2048),
                                        (1100, 900, 64), (129, 0, 128), (257, 1, 129)])
def test_prefill_ragged_shapes(T, off, topk):
    # ragged query groups, partial key tiles, chunk offsets, topk above the
    # visible count (rows return every visible key) and topk = 1
    x = make_prefill("causal_16k_h64", T_q=T - off, T_k=T, q_offset=off, seed=1000 + T)
    check_prefill(x, topk, label=f"T{T} off{off} k{topk}")


def test_prefill_compaction_long_rows():
    # 20k visible keys per row with topk 256: the candidate buffers (3k
    # records) must be compacted many times inside the kernel
    x = make_prefill("causal_16k_h64", T_q=20, T_k=20020, q_offset=20000, seed=77)
    check_prefill(x, 256, label="long rows")
    xh = make_prefill("chunk_128k_h32", T_q=9, T_k=30009, q_offset=30000, seed=78)
    check_prefill(xh, 300, label="long rows H32")


@pytest.mark.parametrize("wl", ["causal_16k_h64", "chunk_128k_h32"])
def test_prefill_two_warpgroup_epilogue(wl):
    # many keys per selected record (150k keys per row split over 25-50
    # CTAs, topk 1: 3000-6000 keys per unit and record): the launch takes
    # the two-warpgroup epilogue with the head weights in registers, where
    # the benchmark shapes take the four-warpgroup one
    x = make_prefill(wl, T_q=24, T_k=150024, q_offset=150000, seed=81)
    check_prefill(x, 1, label=f"two warpgroups {wl}")


def _host(a, dtype, pinned):
    t = torch.from_numpy(np.ascontiguousarray(a))
    t = t.view(torch.int16).view(torch.bfloat16) if dtype == torch.bfloat16 else t
    return t.pin_memory() if pinned else t


@pytest.mark.parametrize("wl,T_q,off,topk,pinned", [("causal_16k_h64", 5000, 100, 256, True),
                                                    ("chunk_128k_h32", 37, 3000, 64, False),
                                                    ("causal_16k_h64", 16384, 0, 2048, True)])
def test_prefill_host_buffers_match_device_call(wl, T_q, off, topk, pinned):
    # host inputs and outputs, rows streamed in blocks through two device
    # slots (ragged last block; one block; eight blocks at the benchmark's
    # size): bit for bit the device call's result, twice in a row
    x = make_prefill(wl, T_q=T_q, T_k=off + T_q, q_offset=off, seed=900 + T_q)
    di, ds = run_prefill(x, topk)
    hq, hw, hk = _host(x["q"].view(np.int16), torch.bfloat16, pinned), _host(x["w"], torch.float32, pinned), \
        _host(x["k"].view(np.int16), torch.bfloat16, pinned)
    ws = torch.empty(dsa.dsa_index_prefill_host_workspace_bytes(T_q, off + T_q, x["H"], 128, topk),
                     dtype=torch.uint8, device="cuda")
    for _ in range(2):
        hi, hs = dsa.dsa_index_prefill_host(hq, hw, hk, off, topk, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(hi.numpy(), di)
        assert np.array_equal(hs.numpy().view(np.uint32), ds.view(np.uint32))
    assert dsa.dsa_index_device_status(ws) == 0


def test_prefill_host_rejects_device_tensors():
    x = make_prefill("causal_16k_h64", T_q=8, T_k=8, q_offset=0, seed=3)
    q = _host(x["q"].view(np.int16), torch.bfloat16, False)
    with pytest.raises(ValueError):
        dsa.dsa_index_prefill_host(q.cuda(), _host(x["w"], torch.float32, False),
                                   _host(x["k"].view(np.int16), torch.bfloat16, False), 0, 4)


def test_non_finite_inputs_set_the_status_bit():
    # a NaN key or an inf query entry inside the causal window sets status
    # bit 3; a NaN in a key no row can see leaves the status clean
    def status_after(q, k, off=0):
        ws = torch.empty(dsa.dsa_index_prefill_workspace_bytes(q.shape[0], k.shape[0], 64, 128, 16),
                         dtype=torch.uint8, device="cuda")
        dsa.dsa_index_prefill(bf16(q), f32(x["w"]), bf16(k), off, 16, workspace=ws)
        return dsa.dsa_index_device_status(ws)
    x = make_prefill("causal_16k_h64", T_q=32, T_k=64, q_offset=0, seed=11)
    assert status_after(x["q"], x["k"]) == 0
    k = x["k"].copy()
    k[10, 5] = 0x7FC0  # bf16 NaN, visible to rows 10..31
    assert status_after(x["q"], k) & 8
    q = x["q"].copy()
    q[3, 7, 0] = 0x7F80  # bf16 +inf in one head of row 3
    assert status_after(q, x["k"]) & 8
    k = x["k"].copy()
    k[50, 0] = 0x7FC0  # past every row's causal window
    assert status_after(x["q"], k) == 0


def test_prefill_key_splits_for_few_rows():
    # 8 query rows against 40k keys: few groups, so each group's keys are
    # split across CTAs and merged by the final selection
    x = make_prefill("chunk_1m_h64", T_q=8, T_k=40008, q_offset=40000, seed=5)
    check_prefill(x, 2048, label="splits")


def test_prefill_integer_ties():
    # small integer inputs produce many exactly tied scores (and exact zeros):
    # ties must come out in ascending key order with identical scores
    x = make_integer_prefill(3, 600, 64, 128, lo=-1, hi=1)
    x["q"] = x["q"].reshape(600, 64, 128)
    gi, gs = run_prefill(x, 50)
    idx, sc, amax = __import__("oracle").prefill_topk(x["q"], x["w"], x["k"], 0, 50)
    # integer inputs: every dot and score is exact in fp32 as well
    assert (gi == idx).all()
    assert (gs.astype(np.float64)[gi >= 0] == sc[gi >= 0]).all()


def test_prefill_rejects_bad_arguments():
    x = make_prefill("causal_1k_h64", T_q=4, T_k=8, q_offset=4)
    q, w, k = bf16(x["q"]), f32(x["w"]), bf16(x["k"])
    with pytest.raises(dsa.DSAError, match="EUNSUPPORTED"):
        dsa.dsa_index_prefill(q, w, k, 4, 4096)
    with pytest.raises(dsa.DSAError, match="EINVAL"):
        dsa.dsa_index_prefill(q, w, k, 5, 8)  # q_offset + T_q > T_k
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(dsa.DSAError, match="EWORKSPACE"):
        dsa.dsa_index_prefill(q, w, k, 4, 8, workspace=ws)


def test_decode_ragged_lengths():
    lens = [3000, 1, 0, 129, 2048, 2049, 128, 2500]
    x = make_decode("decode_64x128k_h64", B=len(lens), t_cap=3000, seq_len=lens, seed=11)
    for topk in (2048, 256, 1):
        idx, sc = dsa.dsa_index_decode(bf16(x["q"]), f32(x["w"]), bf16(x["k"]),
                                       torch.from_numpy(x["seq_len"]).cuda(), topk)
        torch.cuda.synchronize()
        oi, osc, amax, score_of = oracle_decode_rows(x, topk)
        check_rows(idx.cpu().numpy(), sc.cpu().numpy(), oi, osc, amax, x["seq_len"], topk,
                   score_of, f"decode k{topk}")


def test_decode_h32_ragged_lengths():
    # the H = 32 decode kernel (the 128K chunk recipe's heads), ragged caches
    lens = [2500, 0, 1, 1300, 2047, 700]
    x = make_decode("chunk_128k_h32", B=len(lens), t_cap=2500, seq_len=lens, seed=13)
    assert x["H"] == 32
    for topk in (2048, 100):
        idx, sc = dsa.dsa_index_decode(bf16(x["q"]), f32(x["w"]), bf16(x["k"]),
                                       torch.from_numpy(x["seq_len"]).cuda(), topk)
        torch.cuda.synchronize()
        oi, osc, amax, score_of = oracle_decode_rows(x, topk)
        check_rows(idx.cpu().numpy(), sc.cpu().numpy(), oi, osc, amax, x["seq_len"], topk,
                   score_of, f"decode H32 k{topk}")


def test_decode_long_caches_split_across_ctas():
    # few sequences with long caches: each sequence's tiles spread over many
    # CTAs, whose partial candidate lists the final selection merges
    lens = [60000, 33333, 5]
    x = make_decode("decode_64x128k_h64", B=3, t_cap=60000, seq_len=lens, seed=12)
    idx, sc = dsa.dsa_index_decode(bf16(x["q"]), f32(x["w"]), bf16(x["k"]),
                                   torch.from_numpy(x["seq_len"]).cuda(), 2048)
    torch.cuda.synchronize()
    oi, osc, amax, score_of = oracle_decode_rows(x, 2048)
    check_rows(idx.cpu().numpy(), sc.cpu().numpy(), oi, osc, amax, x["seq_len"], 2048, score_of,
               "decode long")


def test_device_status_clean_after_calls():
    x = make_prefill("causal_1k_h64", T_q=64, T_k=64, q_offset=0)
    ws = torch.empty(dsa.dsa_index_prefill_workspace_bytes(64, 64, 64, 128, 16), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_index_prefill(bf16(x["q"]), f32(x["w"]), bf16(x["k"]), 0, 16, workspace=ws)
    assert dsa.dsa_index_device_status(ws) == 0


def test_prefill_row_blocks_match_one_launch():
    # a workspace smaller than the chunk needs: the call runs consecutive
    # launches over row blocks; rows are independent, so the output equals
    # the single-launch output bit for bit
    T_q, off, topk = 3000, 1000, 256
    x = make_prefill("causal_16k_h64", T_q=T_q, T_k=off + T_q, q_offset=off, seed=71)
    q, w, k = bf16(x["q"]), f32(x["w"]), bf16(x["k"])
    full_idx, full_sc = dsa.dsa_index_prefill(q, w, k, off, topk)
    small = dsa.dsa_index_prefill_workspace_bytes(700, off + T_q, 64, 128, topk)
    assert small < dsa.dsa_index_prefill_workspace_bytes(T_q, off + T_q, 64, 128, topk)
    ws = torch.empty(small, dtype=torch.uint8, device="cuda")
    idx, sc = dsa.dsa_index_prefill(q, w, k, off, topk, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(idx, full_idx) and torch.equal(sc.view(torch.int32), full_sc.view(torch.int32))
    assert dsa.dsa_index_device_status(ws) == 0
    # a workspace below one query group is refused
    with pytest.raises(dsa.DSAError, match="EWORKSPACE"):
        dsa.dsa_index_prefill(q, w, k, off, topk, workspace=torch.empty(1 << 16, dtype=torch.uint8, device="cuda"))


# ---------------------------------------------------------------- full sizes

def _sample_rows(T_q, n):
    return np.unique(np.linspace(0, T_q - 1, n).round().astype(np.int64))


@pytest.mark.parametrize("name,n_rows", [("causal_16k_h64", 12), ("chunk_128k_h32", 8),
                                         ("chunk_1m_h64", 6)])
def test_full_size_prefill_sampled_rows(name, n_rows):
    # the benchmark's workloads in the benchmark's launch configuration,
    # checked on evenly spaced rows (first and last included)
    x = make_prefill(name)
    wl = WORKLOADS[name]
    rows = _sample_rows(wl.T_q, n_rows)
    check_prefill(x, wl.topk, rows=rows, label=name)


def test_full_size_decode_sampled_sequences():
    wl = WORKLOADS["decode_64x128k_h64"]
    x = make_decode(wl)
    idx, sc = dsa.dsa_index_decode(bf16(x["q"]), f32(x["w"]), bf16(x["k"]),
                                   torch.from_numpy(x["seq_len"]).cuda(), wl.topk)
    torch.cuda.synchronize()
    pick = np.array([0, 31, 63])
    sub = dict(q=x["q"][pick], w=x["w"][pick], k=x["k"][pick], seq_len=x["seq_len"][pick])
    oi, osc, amax, score_of = oracle_decode_rows(sub, wl.topk)
    check_rows(idx.cpu().numpy()[pick], sc.cpu().numpy()[pick], oi, osc, amax, sub["seq_len"],
               wl.topk, score_of, "decode full")


def test_full_size_32k_row_chunk_against_1m_keys_in_row_blocks():
    # a 32K-row chunk at the end of a 1M context with a 512 MiB workspace:
    # the call runs in row blocks; sampled rows match the oracle
    T_q, T_k = 32768, 1 << 20
    x = make_prefill("chunk_1m_h64", T_q=T_q, T_k=T_k, q_offset=T_k - T_q, seed=72)
    ws = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    idx, sc = dsa.dsa_index_prefill(bf16(x["q"]), f32(x["w"]), bf16(x["k"]), x["q_offset"], 2048, workspace=ws)
    torch.cuda.synchronize()
    assert dsa.dsa_index_device_status(ws) == 0
    rows = _sample_rows(T_q, 5)
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, 2048)
    check_rows(idx.cpu().numpy()[rows], sc.cpu().numpy()[rows], oi, osc, amax, x["q_offset"] + rows + 1, 2048,
               score_of, "32K rows x 1M keys")
