"""Batched decode over a paged key cache (dsa_index_decode_paged).

A sequence's keys live in fixed-size pages of one pool, listed by its block
table.  The result must equal the contiguous-cache decode on the same keys
bit for bit (same tiles, same arithmetic), and match the oracle on the
gathered caches.
"""

import numpy as np
import pytest
import torch

import sparse_attention_token_03_b200 as dsa
from synth import make_decode
from tests.parity import check_rows, oracle_decode_rows

pytestmark = pytest.mark.gpu


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def paged_layout(x, page, seed, spare_pages=3):
    """Scatter every sequence's cache over a shuffled page pool; returns the
    pool (n_pages, page, d) and the block tables (B, max_blocks)."""
    B, t_cap, d = x["k"].shape
    max_blocks = (t_cap + page - 1) // page
    n_pages = B * max_blocks + spare_pages
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n_pages)[:B * max_blocks].reshape(B, max_blocks).astype(np.int32)
    pool = rng.integers(0, 2 ** 15, size=(n_pages, page, d)).astype(np.uint16)  # unused pages: junk
    padded = np.zeros((B, max_blocks * page, d), np.uint16)
    padded[:, :t_cap] = x["k"]
    for b in range(B):
        pool[perm[b]] = padded[b].reshape(max_blocks, page, d)
    return pool, perm


@pytest.mark.parametrize("page", [64, 256])
def test_paged_decode_equals_contiguous_decode_and_oracle(page):
    lens = [3000, 1, 0, 129, 2048, 2049, 128, 2500, 64, 65]
    x = make_decode("decode_64x128k_h64", B=len(lens), t_cap=3000, seq_len=lens, seed=61)
    pool, bt = paged_layout(x, page, seed=62)
    q, w = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda()
    sl = torch.from_numpy(x["seq_len"]).cuda()
    for topk in (2048, 100):
        ci, cs = dsa.dsa_index_decode(q, w, _bf16(x["k"]), sl, topk)
        pi, ps = dsa.dsa_index_decode_paged(q, w, _bf16(pool), torch.from_numpy(bt).cuda(), sl, topk)
        torch.cuda.synchronize()
        assert torch.equal(pi, ci) and torch.equal(ps.view(torch.int32), cs.view(torch.int32))
        oi, osc, amax, score_of = oracle_decode_rows(x, topk)
        check_rows(pi.cpu().numpy(), ps.cpu().numpy(), oi, osc, amax, x["seq_len"], topk, score_of,
                   f"paged {page} k{topk}")


def test_paged_decode_flags_a_bad_page_id():
    x = make_decode("decode_64x128k_h64", B=2, t_cap=256, seq_len=[256, 100], seed=63)
    pool, bt = paged_layout(x, 64, seed=64)
    bt[1, 0] = -5  # a page id outside the pool, in a block holding visible keys
    ws = torch.empty(dsa.dsa_index_decode_workspace_bytes(2, bt.shape[1] * 64, 64, 128, 16), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_index_decode_paged(_bf16(x["q"]), torch.from_numpy(x["w"]).cuda(), _bf16(pool),
                               torch.from_numpy(bt).cuda(), torch.from_numpy(x["seq_len"]).cuda(), 16,
                               workspace=ws)
    assert dsa.dsa_index_device_status(ws) & 2


def test_paged_decode_long_caches_match_contiguous():
    # three long sequences in 64-key pages: each sequence's tiles spread over
    # many CTAs; the paged and contiguous results are identical
    lens = [60000, 33333, 5]
    x = make_decode("decode_64x128k_h64", B=3, t_cap=60000, seq_len=lens, seed=65)
    pool, bt = paged_layout(x, 64, seed=66)
    q, w, sl = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda(), torch.from_numpy(x["seq_len"]).cuda()
    ci, cs = dsa.dsa_index_decode(q, w, _bf16(x["k"]), sl, 2048)
    pi, ps = dsa.dsa_index_decode_paged(q, w, _bf16(pool), torch.from_numpy(bt).cuda(), sl, 2048)
    torch.cuda.synchronize()
    assert torch.equal(pi, ci) and torch.equal(ps.view(torch.int32), cs.view(torch.int32))


def sequence_pages(k, page, seed, spare_pages=2):
    """One sequence's keys (T_k, d) scattered over a shuffled page pool;
    returns the pool (n_pages, page, d) and the block table (n_blocks,)."""
    T_k, d = k.shape
    n_blocks = (T_k + page - 1) // page
    n_pages = n_blocks + spare_pages
    rng = np.random.default_rng(seed)
    bt = rng.permutation(n_pages)[:n_blocks].astype(np.int32)
    pool = rng.integers(0, 2 ** 15, size=(n_pages, page, d)).astype(np.uint16)  # unused pages: junk
    padded = np.zeros((n_blocks * page, d), np.uint16)
    padded[:T_k] = k
    pool[bt] = padded.reshape(n_blocks, page, d)
    return pool, bt


@pytest.mark.parametrize("page,T_q,T_k", [(64, 700, 2500), (16, 300, 1000), (1000, 512, 3000)])
def test_paged_prefill_equals_contiguous(page, T_q, T_k):
    from synth import make_prefill
    x = make_prefill("causal_16k_h64", T_q=T_q, T_k=T_k, q_offset=T_k - T_q, seed=71)
    pool, bt = sequence_pages(x["k"], page, seed=72)
    q, w = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda()
    for topk in (2048, 77):
        ci, cs = dsa.dsa_index_prefill(q, w, _bf16(x["k"]), T_k - T_q, topk)
        pi, ps = dsa.dsa_index_prefill_paged(q, w, _bf16(pool), torch.from_numpy(bt).cuda(), T_k - T_q, topk)
        torch.cuda.synchronize()
        assert torch.equal(pi, ci) and torch.equal(ps.view(torch.int32), cs.view(torch.int32))


def test_paged_prefill_row_blocks_in_a_small_workspace():
    # a workspace below the full size: the keys are gathered once and the
    # rows run in blocks; the result is unchanged
    from synth import make_prefill
    T_q = T_k = 4096
    x = make_prefill("causal_16k_h64", T_q=T_q, T_k=T_k, q_offset=0, seed=73)
    pool, bt = sequence_pages(x["k"], 128, seed=74)
    q, w = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda()
    full = dsa.dsa_index_prefill_paged_workspace_bytes(T_q, T_k, 64, 128, 2048)
    ws = torch.empty(full // 3, dtype=torch.uint8, device="cuda")
    ci, cs = dsa.dsa_index_prefill(q, w, _bf16(x["k"]), 0, 2048)
    pi, ps = dsa.dsa_index_prefill_paged(q, w, _bf16(pool), torch.from_numpy(bt).cuda(), 0, 2048, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(pi, ci) and torch.equal(ps.view(torch.int32), cs.view(torch.int32))


def test_paged_pruned_equals_contiguous_pruned():
    from synth import make_prefill, random_distinct_keys
    T_k, T_q, topk = 6000, 512, 512
    x = make_prefill("chunk_128k_h32", T_q=T_q, T_k=T_k, q_offset=T_k - T_q, seed=75)
    pool, bt = sequence_pages(x["k"], 64, seed=76)
    seeds = torch.from_numpy(random_distinct_keys(77, 0, T_k - T_q, 1536)).cuda()
    q, w = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda()
    ci, cs, cst = dsa.dsa_index_prefill_pruned(q, w, _bf16(x["k"]), T_k - T_q, topk, seeds, stats=True)
    pi, ps, pst = dsa.dsa_index_prefill_pruned_paged(q, w, _bf16(pool), torch.from_numpy(bt).cuda(), T_k - T_q,
                                                     topk, seeds, stats=True)
    di, ds = dsa.dsa_index_prefill(q, w, _bf16(x["k"]), T_k - T_q, topk)
    torch.cuda.synchronize()
    assert torch.equal(pi, ci) and torch.equal(ps.view(torch.int32), cs.view(torch.int32))
    assert torch.equal(pi, di) and torch.equal(ps.view(torch.int32), ds.view(torch.int32))
    assert pst == cst


def test_paged_prefill_flags_a_bad_page_id():
    from synth import make_prefill
    x = make_prefill("causal_16k_h64", T_q=256, T_k=1024, q_offset=768, seed=78)
    pool, bt = sequence_pages(x["k"], 64, seed=79)
    bt[3] = pool.shape[0] + 7  # outside the pool
    q, w = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda()
    ws = torch.empty(dsa.dsa_index_prefill_paged_workspace_bytes(256, 1024, 64, 128, 64), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_index_prefill_paged(q, w, _bf16(pool), torch.from_numpy(bt).cuda(), 768, 64, workspace=ws)
    assert dsa.dsa_index_device_status(ws) & 2
