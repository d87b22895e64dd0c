"""Failure handling on the GPU, injected on the host (nothing faults or hangs).

Every wait inside the library's kernels is bounded.  A one-shot injection
(dsa_test_inject_wait_timeout) makes the next scoring launch withhold its
loads, so its MMA warp waits for data that never arrives: the wait gives up
after a short limit, the kernel unwinds, the device status word carries the
timeout bit, a synchronous call reports DSA_EDEVICE, and the next call on the
same device is exact again ("DoSA" reading notes, annotation TMIF4XYF: errors
leave an exact path to recover through).
"""

import numpy as np
import pytest
import torch

import sparse_attention_token_03_b200 as dsa
from synth import make_prefill, random_distinct_keys
from tests.parity import check_rows, oracle_prefill_rows

pytestmark = pytest.mark.gpu

LIMIT_NS = 50_000_000  # 50 ms


def _dev(x):
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    return bf(x["q"]), torch.from_numpy(x["w"]).cuda(), bf(x["k"])


@pytest.mark.parametrize("wl,H", [("causal_1k_h64", 64), ("chunk_128k_h32", 32)])
def test_injected_wait_timeout_sets_the_status_and_the_next_call_is_exact(wl, H):
    off, T_q, topk = 536, 64, 32
    x = make_prefill(wl, T_q=T_q, T_k=off + T_q, q_offset=off, seed=41)
    q, w, k = _dev(x)
    ws = torch.zeros(dsa.dsa_index_prefill_workspace_bytes(T_q, off + T_q, H, 128, topk), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_test_inject_wait_timeout(LIMIT_NS)
    dsa.dsa_index_prefill(q, w, k, off, topk, workspace=ws)
    torch.cuda.synchronize()
    assert dsa.dsa_index_device_status(ws) & 1, "the timeout bit must be set"
    # the context is still usable and the next call is exact
    idx, sc = dsa.dsa_index_prefill(q, w, k, off, topk, workspace=ws)
    torch.cuda.synchronize()
    assert dsa.dsa_index_device_status(ws) == 0
    rows = np.arange(T_q)
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, topk)
    check_rows(idx.cpu().numpy(), sc.cpu().numpy(), oi, osc, amax, off + rows + 1, topk, score_of, "after timeout")


def test_injected_wait_timeout_makes_the_synchronous_pruned_call_fail():
    off, T_q, topk = 536, 64, 32
    x = make_prefill("causal_1k_h64", T_q=T_q, T_k=off + T_q, q_offset=off, seed=42)
    q, w, k = _dev(x)
    seeds = torch.from_numpy(random_distinct_keys(43, 0, off, 96)).cuda()
    ws = torch.zeros(dsa.dsa_index_prefill_pruned_workspace_bytes(T_q, off + T_q, 64, 128, topk, 96),
                     dtype=torch.uint8, device="cuda")
    dsa.dsa_test_inject_wait_timeout(LIMIT_NS)
    with pytest.raises(dsa.DSAError, match="EDEVICE"):
        dsa.dsa_index_prefill_pruned(q, w, k, off, topk, seeds, workspace=ws, stats=True)
    pi, ps, st = dsa.dsa_index_prefill_pruned(q, w, k, off, topk, seeds, workspace=ws, stats=True)
    di, ds = dsa.dsa_index_prefill(q, w, k, off, topk)
    torch.cuda.synchronize()
    assert torch.equal(pi, di) and torch.equal(ps, ds)


def test_injection_limit_is_validated_on_the_host():
    with pytest.raises(dsa.DSAError, match="EINVAL"):
        dsa.dsa_test_inject_wait_timeout(10)
