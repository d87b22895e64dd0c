"""The allocation-free decode entry point (dsa_index_decode_noalloc).

Some callers cannot give the library device memory (their device memory is
owned by an allocator they cannot reach, or a cudaMalloc would stall a
latency-critical path), so this entry point runs the decode path out of a
fixed scratch array inside the library.  Its results must match the regular
workspace-based decode, call after call, since every call reuses (and must
re-initialise) the same scratch.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import sparse_attention_token_03_b200 as dsa
from synth import make_decode

pytestmark = pytest.mark.gpu


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("topk", [2048, 100])
def test_noalloc_decode_matches_workspace_decode_twice(topk):
    lens = [3000, 1, 0, 129, 2048, 2049, 128, 2999]
    x = make_decode("decode_64x128k_h64", B=len(lens), t_cap=3000, seq_len=lens, seed=31)
    q, w, k = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda(), _bf16(x["k"])
    sl = torch.from_numpy(x["seq_len"]).cuda()
    ref_idx, ref_sc = dsa.dsa_index_decode(q, w, k, sl, topk)
    out_idx = torch.empty_like(ref_idx)
    out_sc = torch.empty_like(ref_sc)
    for _ in range(2):
        out_idx.fill_(-7)
        out_sc.fill_(float("nan"))
        dsa.dsa_index_decode_noalloc(q, w, k, sl, topk, out_idx=out_idx, out_score=out_sc)
        torch.cuda.synchronize()
        assert torch.equal(out_idx, ref_idx)
        # same kernels, same arithmetic: the scores agree far inside the
        # parity tolerance (2e-3 of the row's largest |score|); checked exactly
        assert torch.equal(out_sc, ref_sc)
        torch.testing.assert_close(out_sc, ref_sc, rtol=0, atol=0)


def test_noalloc_decode_rejects_batches_above_its_static_limit():
    x = make_decode("decode_64x128k_h64", B=65, t_cap=16, seed=32)
    q, w, k = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda(), _bf16(x["k"])
    sl = torch.from_numpy(x["seq_len"]).cuda()
    with pytest.raises(dsa.DSAError, match="static scratch limit"):
        dsa.dsa_index_decode_noalloc(q, w, k, sl, 8)


def test_noalloc_decode_reports_device_checks_in_its_own_status_word():
    # the static scratch carries the device status word: a length above the
    # cache capacity is treated as 0 and sets bit 1, readable without a
    # workspace; the next clean call clears it
    lens = [40, 17]
    x = make_decode("decode_64x128k_h64", B=2, t_cap=40, seq_len=lens, seed=33)
    q, w, k = _bf16(x["q"]), torch.from_numpy(x["w"]).cuda(), _bf16(x["k"])
    bad = torch.tensor([40, 41], dtype=torch.int32, device="cuda")  # 41 > t_cap
    idx, _ = dsa.dsa_index_decode_noalloc(q, w, k, bad, 8)
    torch.cuda.synchronize()
    assert dsa.dsa_index_decode_noalloc_status() & 2
    assert (idx[1] == -1).all().item()  # the bad sequence sees no keys
    sl = torch.from_numpy(x["seq_len"]).cuda()
    dsa.dsa_index_decode_noalloc(q, w, k, sl, 8)
    assert dsa.dsa_index_decode_noalloc_status() == 0
