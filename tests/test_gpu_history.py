"""Seeds from historical selection frequency (dsa_index_seeds_from_history).

Integer work: the GPU's seed list must equal the oracle's bit for bit (the
n_seed most selected keys, ties to the smaller key, in ascending order).  The
end-to-end case feeds one chunk's Top-k lists to the next chunk's pruned
prefill, whose output must still equal the dense path's.
"""

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_03_b200 as dsa
from synth import make_prefill

pytestmark = pytest.mark.gpu


def history(rng, n_rows, topk, n_keys, zipf=1.3, pad=0.0):
    """Rows of distinct keys drawn with Zipf-like popularity, -1 padded."""
    rows = np.empty((n_rows, topk), np.int32)
    for r in range(n_rows):
        pick = np.unique(np.minimum(rng.zipf(zipf, 3 * topk) - 1, n_keys - 1))
        pick = pick[rng.permutation(pick.shape[0])]
        extra = rng.choice(n_keys, size=topk, replace=False)
        row = np.concatenate([pick, extra[~np.isin(extra, pick)]])[:topk]
        n_pad = int(pad * topk)
        if n_pad:
            row[topk - n_pad:] = -1
        rows[r] = row
    return rows


def gpu_seeds(prev, n_keys, n_seed):
    out = dsa.dsa_index_seeds_from_history(torch.from_numpy(prev).cuda(), n_keys, n_seed)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("n_rows,topk,n_keys,n_seed,pad", [
    (64, 256, 4096, 1024, 0.0),          # a few tiles
    (300, 512, 100_003, 6144, 0.25),     # ragged last tile, padding
    (1024, 2048, 131_072, 12_288, 0.0),  # the long-context seed size
    (16, 64, 1000, 1000, 0.0),           # every key a seed
    (16, 64, 5000, 1, 0.0),              # one seed
])
def test_history_seeds_match_oracle(n_rows, topk, n_keys, n_seed, pad):
    rng = np.random.default_rng(n_keys + n_seed)
    prev = history(rng, n_rows, topk, n_keys, pad=pad)
    want, _ = oracle.seeds_from_history(prev, n_keys, n_seed)
    got = gpu_seeds(prev, n_keys, n_seed)
    np.testing.assert_array_equal(got, want)


def test_history_seeds_out_of_range_and_large_counts():
    """Keys at or beyond n_keys are not counted; counts above 2^16 exercise
    the high half of the radix cut-off."""
    rng = np.random.default_rng(7)
    n_keys = 50_000
    prev = rng.integers(-3, n_keys + 500, size=(70_000, 4)).astype(np.int32)
    prev[:, 0] = 17          # count 70000 > 65535
    prev[:66_000, 1] = 4242  # count >= 66000
    want, counts = oracle.seeds_from_history(prev, n_keys, 3000)
    assert counts[17] >= 70_000 and counts[4242] >= 66_000
    np.testing.assert_array_equal(gpu_seeds(prev, n_keys, 3000), want)


def test_history_seeds_empty_history():
    got = dsa.dsa_index_seeds_from_history(torch.empty((0, 8), dtype=torch.int32, device="cuda"), 300, 37)
    np.testing.assert_array_equal(got.cpu().numpy(), np.arange(37, dtype=np.int32))


def test_history_seeds_rejects_bad_sizes():
    prev = torch.zeros((4, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(dsa.DSAError):
        dsa.dsa_index_seeds_from_history(prev, 10, 11)
    with pytest.raises(dsa.DSAError):
        dsa.dsa_index_seeds_from_history(prev, 10, 0)


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def test_history_seeds_feed_next_chunk_exactly():
    """Chunk A's dense Top-k lists give chunk B's seeds; B's pruned output is
    the dense output bit for bit."""
    C, T_k, topk = 2048, 32768, 2048
    x = make_prefill("chunk_128k_h32", T_q=2 * C, T_k=T_k, q_offset=T_k - 2 * C, seed=11)
    q, w, k = bf16(x["q"]), torch.from_numpy(x["w"]).cuda(), bf16(x["k"])
    off_a, off_b = T_k - 2 * C, T_k - C
    ia, _ = dsa.dsa_index_prefill(q[:C], w[:C], k[:off_b], off_a, topk)
    seeds = dsa.dsa_index_seeds_from_history(ia, off_b, 3 * topk)
    want_seeds, _ = oracle.seeds_from_history(ia.cpu().numpy(), off_b, 3 * topk)
    np.testing.assert_array_equal(seeds.cpu().numpy(), want_seeds)
    di, ds = dsa.dsa_index_prefill(q[C:], w[C:], k, off_b, topk)
    pi, ps, st = dsa.dsa_index_prefill_pruned(q[C:], w[C:], k, off_b, topk, seeds, stats=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(pi.cpu().numpy(), di.cpu().numpy())
    np.testing.assert_array_equal(ps.cpu().numpy(), ds.cpu().numpy())
    print(f"history-seeded chunk: {st}")
