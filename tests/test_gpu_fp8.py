"""The FP8 (E4M3) prefill (dsa_index_prefill_fp8) against the fp64 FP8 oracle.

Inputs are the bf16 recipes quantised per row to E4M3 codes with fp32
scales; the oracle scores the scaled E4M3 values in fp64 ("DeepSeek DSA
FLOPs", Lightning Indexer: the indexer runs in FP8).  Same tolerance and tie
rule as the bf16 parity tests (tests/parity.py).
"""

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_03_b200 as dsa
from synth import WORKLOADS, make_prefill_fp8
from tests.parity import check_rows

pytestmark = pytest.mark.gpu


def _dev(x):
    u8 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return u8(x["q8"]), f32(x["q_scale"]), f32(x["w"]), u8(x["k8"]), f32(x["k_scale"])


def check_fp8(x, topk, rows=None, label="", workspace=None):
    T_q = x["q8"].shape[0]
    rows = np.arange(T_q) if rows is None else np.asarray(rows)
    idx, sc = dsa.dsa_index_prefill_fp8(*_dev(x), x["q_offset"], topk, workspace=workspace)
    torch.cuda.synchronize()
    gi, gs = idx.cpu().numpy()[rows], sc.cpu().numpy()[rows]
    oi, osc, amax = oracle.prefill_topk_fp8(x["q8"], x["q_scale"], x["w"], x["k8"], x["k_scale"],
                                             x["q_offset"], topk, rows=rows)

    def score_of(i, keys):
        r = np.full(len(keys), rows[i], np.int64)
        return oracle.score_pairs_fp8(x["q8"], x["q_scale"], x["w"], x["k8"], x["k_scale"], r, keys)

    return check_rows(gi, gs, oi, osc, amax, x["q_offset"] + rows + 1, topk, score_of, label)


@pytest.mark.parametrize("recipe,H", [("causal_1k_h64", 64), ("chunk_128k_h32", 32)])
def test_fp8_prefill_tiny_full_causal(recipe, H):
    x = make_prefill_fp8(recipe, T_q=1024, T_k=1024, q_offset=0, seed=51)
    assert x["H"] == H
    check_fp8(x, 256, label=f"fp8 causal1k H{H}")


@pytest.mark.parametrize("T,off,topk", [(1, 0, 1), (37, 0, 5), (300, 123, 2048), (1100, 900, 64),
                                        (257, 1, 129)])
def test_fp8_prefill_ragged_shapes(T, off, topk):
    x = make_prefill_fp8("causal_16k_h64", T_q=T - off, T_k=T, q_offset=off, seed=2000 + T)
    check_fp8(x, topk, label=f"fp8 T{T} off{off} k{topk}")


def test_fp8_prefill_long_rows_and_key_splits():
    # compactions inside the kernel, and few rows whose keys split over CTAs
    x = make_prefill_fp8("causal_16k_h64", T_q=20, T_k=20020, q_offset=20000, seed=52)
    check_fp8(x, 256, label="fp8 long rows")
    x = make_prefill_fp8("chunk_1m_h64", T_q=8, T_k=40008, q_offset=40000, seed=53)
    check_fp8(x, 2048, label="fp8 splits")


def test_fp8_prefill_row_blocks_match_one_launch():
    T_q, off, topk = 3000, 1000, 256
    x = make_prefill_fp8("chunk_128k_h32", T_q=T_q, T_k=off + T_q, q_offset=off, seed=54)
    full = dsa.dsa_index_prefill_fp8(*_dev(x), off, topk)
    ws = torch.empty(dsa.dsa_index_prefill_workspace_bytes(700, off + T_q, 32, 128, topk), dtype=torch.uint8,
                     device="cuda")
    blk = dsa.dsa_index_prefill_fp8(*_dev(x), off, topk, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(full[0], blk[0]) and torch.equal(full[1].view(torch.int32), blk[1].view(torch.int32))
    assert dsa.dsa_index_device_status(ws) == 0


@pytest.mark.parametrize("name,n_rows", [("causal_16k_h64", 8), ("chunk_128k_h32", 5)])
def test_fp8_full_size_sampled_rows(name, n_rows):
    wl = WORKLOADS[name]
    x = make_prefill_fp8(wl)
    rows = np.unique(np.linspace(0, wl.T_q - 1, n_rows).round().astype(np.int64))
    check_fp8(x, wl.topk, rows=rows, label=f"fp8 {name}")


def test_fp8_accepts_float8_tensors_and_flags_bad_scales():
    x = make_prefill_fp8("causal_16k_h64", T_q=16, T_k=80, q_offset=64, seed=55)
    q8, qs, w, k8, ks = _dev(x)
    a = dsa.dsa_index_prefill_fp8(q8.view(torch.float8_e4m3fn), qs, w, k8.view(torch.float8_e4m3fn), ks, 64, 8)
    b = dsa.dsa_index_prefill_fp8(q8, qs, w, k8, ks, 64, 8)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])
    ws = torch.empty(dsa.dsa_index_prefill_workspace_bytes(16, 80, 64, 128, 8), dtype=torch.uint8, device="cuda")
    bad = ks.clone()
    bad[10] = -1.0  # a negative key scale inside every row's window
    dsa.dsa_index_prefill_fp8(q8, qs, w, k8, bad, 64, 8, workspace=ws)
    assert dsa.dsa_index_device_status(ws) & 8
