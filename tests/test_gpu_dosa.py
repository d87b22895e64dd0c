"""DoSA certified pruning (dsa_index_prefill_pruned) on the GPU.

Its losslessness invariant: on the same inputs the pruned path returns the
dense path's output bit for bit ("DoSA", the pruned selection keeps the
original Top-k).  Both are also checked against the fp64 oracle, and the
recovery paths (bad seeds, survivor overflow) must stay exact.
"""

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_token_03_b200 as dsa
from synth import WORKLOADS, make_prefill, random_distinct_keys
from tests.parity import check_rows, oracle_prefill_rows

pytestmark = pytest.mark.gpu


def bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev_inputs(x):
    return bf16(x["q"]), torch.from_numpy(x["w"]).cuda(), bf16(x["k"])


def anchor_seeds(x, topk, n_random, seed):
    """The recipe of the long-context chunks: the oracle's Top-topk of the
    query just before the chunk, plus distinct random keys before the chunk."""
    off = x["q_offset"]
    qa, wa = x["q_anchor"], x["w_anchor"]
    idx, _, _ = oracle.prefill_topk(qa[None], wa[None], x["k"][:off], off - 1, topk)
    anchor = idx[0][idx[0] >= 0]
    rnd = random_distinct_keys(seed, 0, off, n_random, exclude=anchor)
    return np.concatenate([anchor, rnd]).astype(np.int32)


PROBE_ROWS = 64  # rows of a chunk longer than 128 rows that always take the pruned path


def run_both(x, topk, seeds, workspace=None):
    q, w, k = dev_inputs(x)
    di, ds = dsa.dsa_index_prefill(q, w, k, x["q_offset"], topk)
    pi, ps, st = dsa.dsa_index_prefill_pruned(q, w, k, x["q_offset"], topk,
                                              torch.from_numpy(seeds).cuda(), stats=True,
                                              workspace=workspace)
    torch.cuda.synchronize()
    return di.cpu().numpy(), ds.cpu().numpy(), pi.cpu().numpy(), ps.cpu().numpy(), st


def check_refine_counts(st, all_refined=False):
    """refined_pairs counts the exact scores computed: one per survivor in a
    row's own list, four per key of a group's shared stream (a shared key is
    a survivor of at least two of the group's four rows)."""
    shared = st["shared_keys"]
    assert shared >= 0
    if all_refined:  # no row recovered: every survivor was refined once
        own = st["refined_pairs"] - 4 * shared
        assert own >= 0 and st["survivor_pairs"] > 0
        assert own + 2 * shared <= st["survivor_pairs"] <= own + 4 * shared
    else:
        assert st["refined_pairs"] - 4 * shared <= st["survivor_pairs"]


def screened_rows(T_q, st):
    """Rows that went through the screen: all of them, or only the probe when
    the probe sent the rest of the chunk to the dense pass."""
    if st["bypassed_rows"] == 0:
        return T_q
    assert T_q > 2 * PROBE_ROWS and st["bypassed_rows"] == T_q - PROBE_ROWS
    return PROBE_ROWS


def expected_screened_pairs(off, T_q, n_seed, st):
    n = screened_rows(T_q, st)
    return sum(off + t + 1 - n_seed for t in range(n))


@pytest.mark.parametrize("recipe,H", [("causal_1k_h64", 64), ("causal_16k_h64", 64),
                                      ("chunk_128k_h32", 32), ("chunk_1m_h64", 64)])
def test_pruned_equals_dense_bitwise_and_oracle(recipe, H):
    T_k, off, topk = 1536, 1024, 128
    x = make_prefill(recipe, T_q=T_k - off, T_k=T_k, q_offset=off, seed=404, with_anchor=True)
    seeds = anchor_seeds(x, topk, 200, seed=7)
    di, ds, pi, ps, st = run_both(x, topk, seeds)
    assert np.array_equal(pi, di), "pruned indices differ from the dense path"
    assert np.array_equal(ps.view(np.uint32), ds.view(np.uint32)), "pruned scores differ bitwise"
    rows = np.arange(0, T_k - off, 7)
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, topk)
    check_rows(pi[rows], ps[rows], oi, osc, amax, off + rows + 1, topk, score_of, f"pruned {recipe}")
    T_q = T_k - off
    assert st["screened_pairs"] == expected_screened_pairs(off, T_q, len(seeds), st)
    assert 0 <= st["survivor_pairs"] <= st["screened_pairs"]
    check_refine_counts(st)
    print(recipe, st)


@pytest.mark.parametrize("H", [64, 32])
def test_pruned_refine_path_with_a_tight_bound(H):
    # Heads built so that the bound is exact up to its safety slack: 14
    # distinct heads with large weights (the planner retains them) and H-14
    # identical copies of one vector with small negative weights (no positive
    # omitted head; folding identical negative heads loses nothing).  The 24
    # rows repeat one query and the seeds hold its Top-k among the keys before
    # the chunk, so tau is close to every row's k-th score: nearly every
    # non-Top-k key is pruned and the result comes from screen -> compact ->
    # refine, with no dense recovery.
    T_q, off, topk = 24, 6000, 128
    x = make_prefill("causal_1k_h64" if H == 64 else "chunk_128k_h32", T_q=T_q, T_k=off + T_q,
                     q_offset=off, seed=407)
    rng = np.random.default_rng(0)
    q0 = x["q"][0].copy()
    q0[14:] = q0[14]
    w0 = np.empty(H, np.float32)
    w0[:14] = rng.standard_normal(14).astype(np.float32) * 4.0
    w0[14:] = -0.01
    x["q"][:] = q0
    x["w"][:] = w0
    idx, _, _ = oracle.prefill_topk(x["q"][:1], x["w"][:1], x["k"][:off], off - 1, topk)
    seeds = np.concatenate([idx[0], random_distinct_keys(13, 0, off, 300, exclude=idx[0])]).astype(np.int32)
    di, ds, pi, ps, st = run_both(x, topk, seeds)
    print("tight bound", H, st, "filter rate", 1 - st["survivor_pairs"] / st["screened_pairs"])
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))
    assert st["recovered_rows"] == 0
    check_refine_counts(st, all_refined=True)
    assert st["survivor_pairs"] < 0.2 * st["screened_pairs"]
    assert st["shared_keys"] > 0  # the rows repeat one query: their survivors are shared
    rows = np.array([0, 11, 23])
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, topk)
    check_rows(pi[rows], ps[rows], oi, osc, amax, off + rows + 1, topk, score_of, f"tight {H}")


def test_pruned_filter_rate_on_shared_latent_heads():
    # statistics only (the filter rate depends on the data): heads mixed from
    # one latent row per query, rows repeating one query
    T_q, off, topk = 24, 6000, 128
    x = make_prefill("chunk_1m_h64", T_q=T_q, T_k=off + T_q, q_offset=off, seed=406, head_rank=1)
    x["q"][1:] = x["q"][0]
    x["w"][1:] = x["w"][0]
    idx, _, _ = oracle.prefill_topk(x["q"][:1], x["w"][:1], x["k"][:off], off - 1, topk)
    seeds = np.concatenate([idx[0], random_distinct_keys(13, 0, off, 300, exclude=idx[0])]).astype(np.int32)
    di, ds, pi, ps, st = run_both(x, topk, seeds)
    print("shared latent", st, "filter rate", 1 - st["survivor_pairs"] / st["screened_pairs"])
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))


def test_pruned_ragged_chunk_and_small_topk():
    # a chunk whose rows are not a multiple of any tile or group size
    x = make_prefill("causal_16k_h64", T_q=37, T_k=3037, q_offset=3000, seed=5, with_anchor=True)
    seeds = anchor_seeds(x, 9, 300, seed=8)
    di, ds, pi, ps, st = run_both(x, 9, seeds)
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))


def test_pruned_overflowing_rows_are_recovered_exactly():
    # only topk random seeds: tau is weak, survivors exceed the per-row list
    # (max(T_k/16, 4 topk) = 514 keys), and those rows take the dense path
    x = make_prefill("causal_1k_h64", T_q=40, T_k=8232, q_offset=8192, seed=9)
    seeds = random_distinct_keys(3, 0, 8192, 64)
    di, ds, pi, ps, st = run_both(x, 64, seeds)
    assert st["recovered_rows"] > 0
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))


def test_pruned_bad_seed_lists():
    x = make_prefill("causal_1k_h64", T_q=16, T_k=600, q_offset=584, seed=10)
    q, w, k = dev_inputs(x)
    di, ds = dsa.dsa_index_prefill(q, w, k, 584, 32)
    # fewer seeds than topk: refused before any launch
    with pytest.raises(dsa.DSAError, match="ESEED"):
        dsa.dsa_index_prefill_pruned(q, w, k, 584, 32, torch.arange(31, dtype=torch.int32, device="cuda"))
    # a repeated seed and a seed that is not visible to every row: detected on
    # the device, every row recomputed densely, reported with stats
    for bad in ([5] + list(range(40, 80)) + [5], list(range(0, 40)) + [590]):
        s = torch.tensor(bad, dtype=torch.int32, device="cuda")
        with pytest.raises(dsa.DSAError, match="ESEED"):
            dsa.dsa_index_prefill_pruned(q, w, k, 584, 32, s, stats=True)
        pi, ps = dsa.dsa_index_prefill_pruned(q, w, k, 584, 32, s)
        torch.cuda.synchronize()
        assert torch.equal(pi, di) and torch.equal(ps, ds)


@pytest.mark.parametrize("name,n_rows", [("chunk_128k_h32", 6), ("chunk_1m_h64", 4)])
def test_full_size_pruned_equals_dense(name, n_rows):
    wl = WORKLOADS[name]
    x = make_prefill(wl, with_anchor=True)
    seeds = anchor_seeds(x, wl.topk, wl.n_seed - wl.n_anchor, seed=11)
    assert len(seeds) == wl.n_seed
    di, ds, pi, ps, st = run_both(x, wl.topk, seeds)
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))
    rows = np.unique(np.linspace(0, wl.T_q - 1, n_rows).round().astype(np.int64))
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, wl.topk)
    check_rows(pi[rows], ps[rows], oi, osc, amax, wl.q_offset + rows + 1, wl.topk, score_of, name)
    print(name, st, "filter rate", 1 - st["survivor_pairs"] / st["screened_pairs"])


def _oracle_row_scores(x, row, n_keys):
    return oracle.row_scores(x["q"][row], x["w"][row], x["k"], n_keys)


def check_screen_safety(x, topk, seeds, ws, st, rows):
    """Every key the GPU screen pruned scores (exactly, in fp64) strictly below
    the row's GPU threshold tau ("DoSA", step 2: prune only when the bound is
    below the threshold; the bound never underestimates a score), and tau is
    the row's topk-th seed score up to the parity tolerance."""
    off, T_q, T_k, H = x["q_offset"], x["q"].shape[0], x["k"].shape[0], x["H"]
    mask, tau, state = dsa.dsa_index_prefill_pruned_survivors(ws, T_q, T_k, off, H, 128, topk, len(seeds))
    torch.cuda.synchronize()
    mask = mask.cpu().numpy().view(np.uint32)
    tau, state = tau.cpu().numpy(), state.cpu().numpy()
    is_seed = np.zeros(T_k, bool)
    is_seed[seeds] = True
    checked = 0
    for t in rows:
        assert state[t] in (0, 1), f"row {t} was not screened (state {state[t]})"
        nvis = off + t + 1
        bits = ((mask[t][np.arange(nvis) >> 5] >> (np.arange(nvis) & 31)) & 1).astype(bool)
        assert not (bits & is_seed[:nvis]).any(), "seed keys must not appear as screened survivors"
        I = _oracle_row_scores(x, t, nvis)
        pruned = ~bits & ~is_seed[:nvis]
        worst = float(I[pruned].max()) if pruned.any() else -np.inf
        assert worst < float(tau[t]), f"row {t}: pruned key scores {worst} >= tau {tau[t]}"
        seed_sc = np.sort(I[seeds])[::-1]
        tol = 2e-3 * float(np.abs(I).max())
        assert abs(float(tau[t]) - seed_sc[topk - 1]) <= tol, (t, tau[t], seed_sc[topk - 1])
        checked += int(pruned.sum())
    return checked


@pytest.mark.parametrize("recipe,head_rank", [("causal_1k_h64", 0), ("causal_16k_h64", 1)])
def test_screen_prunes_only_keys_below_tau_tiny_chunk(recipe, head_rank):
    # 1024 keys split at q_offset = 512 (the oracle-sized shape; the shared
    # latent heads let the bound prune): every screened row, every visible
    # key checked against the fp64 scores
    off, T_k, topk = 512, 1024, 256
    x = make_prefill(recipe, T_q=T_k - off, T_k=T_k, q_offset=off, seed=21, head_rank=head_rank)
    seeds = random_distinct_keys(22, 0, off, 384)
    ws = torch.zeros(dsa.dsa_index_prefill_pruned_workspace_bytes(T_k - off, T_k, 64, 128, topk, len(seeds)),
                     dtype=torch.uint8, device="cuda")
    di, ds, pi, ps, st = run_both(x, topk, seeds, workspace=ws)
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))
    n = screened_rows(T_k - off, st)
    pruned = check_screen_safety(x, topk, seeds, ws, st, range(n))
    print("tiny chunk", recipe, head_rank, "pruned keys checked", pruned, st)
    if head_rank:
        assert pruned > 0


@pytest.mark.parametrize("head_rank", [0, 1])
def test_screen_prunes_only_keys_below_tau_full_size_128k(head_rank):
    # the 128K / H32 chunk at full size (8192 rows x 131072 keys, the
    # benchmark's seed recipe); rows spread over the screened ones
    wl = WORKLOADS["chunk_128k_h32"]
    x = make_prefill(wl, with_anchor=True, head_rank=head_rank)
    seeds = anchor_seeds(x, wl.topk, wl.n_seed - wl.n_anchor, seed=11)
    ws = torch.zeros(dsa.dsa_index_prefill_pruned_workspace_bytes(wl.T_q, wl.T_k, wl.H, 128, wl.topk, wl.n_seed),
                     dtype=torch.uint8, device="cuda")
    di, ds, pi, ps, st = run_both(x, wl.topk, seeds, workspace=ws)
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))
    n = screened_rows(wl.T_q, st)
    rows = np.unique(np.linspace(0, n - 1, 6).round().astype(np.int64))
    pruned = check_screen_safety(x, wl.topk, seeds, ws, st, rows)
    print("128K chunk head_rank", head_rank, "pruned keys checked", pruned, st)


def _tight_bound_chunk(wl_name, T_q, T_k, off, topk, seed, n_random):
    """Rows repeating one query built so that the DoSA bound is exact up to its
    safety slack: 14 distinct heads with large weights (the planner retains
    them) and H-14 identical copies of one vector with small negative weights
    (no positive omitted head; folding identical negative heads loses
    nothing).  The seeds hold the query's Top-k among the keys before the
    chunk, so tau is close to every row's k-th score."""
    x = make_prefill(wl_name, T_q=T_q, T_k=T_k, q_offset=off, seed=seed)
    H = x["H"]
    rng = np.random.default_rng(0)
    q0 = x["q"][0].copy()
    q0[14:] = q0[14]
    w0 = np.empty(H, np.float32)
    w0[:14] = rng.standard_normal(14).astype(np.float32) * 4.0
    w0[14:] = -0.01
    x["q"][:] = q0
    x["w"][:] = w0
    idx, _, _ = oracle.prefill_topk(x["q"][:1], x["w"][:1], x["k"][:off], off - 1, topk)
    seeds = np.concatenate([idx[0], random_distinct_keys(13, 0, off, n_random, exclude=idx[0])]).astype(np.int32)
    return x, seeds


def test_full_size_pruned_refine_path_without_recovery():
    # the 128K / H32 chunk's sizes (8192 rows x 131072 keys, 12288 seeds) with
    # the constructed tight-bound heads: the probe keeps the pruned path, no
    # row overflows, the result comes from screen -> compact -> refine and is
    # bit for bit the dense one
    wl = WORKLOADS["chunk_128k_h32"]
    x, seeds = _tight_bound_chunk("chunk_128k_h32", wl.T_q, wl.T_k, wl.q_offset, wl.topk, 408,
                                  wl.n_seed - wl.topk)
    assert len(seeds) == wl.n_seed
    ws = torch.zeros(dsa.dsa_index_prefill_pruned_workspace_bytes(wl.T_q, wl.T_k, wl.H, 128, wl.topk, wl.n_seed),
                     dtype=torch.uint8, device="cuda")
    di, ds, pi, ps, st = run_both(x, wl.topk, seeds, workspace=ws)
    print("full-size tight bound", st, "filter rate", 1 - st["survivor_pairs"] / st["screened_pairs"])
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))
    assert st["bypassed_rows"] == 0 and st["recovered_rows"] == 0
    check_refine_counts(st, all_refined=True)
    assert st["shared_keys"] > 0
    assert st["screened_pairs"] == expected_screened_pairs(wl.q_offset, wl.T_q, wl.n_seed, st)
    rows = np.array([0, 4095, wl.T_q - 1])
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, wl.topk)
    check_rows(pi[rows], ps[rows], oi, osc, amax, wl.q_offset + rows + 1, wl.topk, score_of, "tight full")
    check_screen_safety(x, wl.topk, seeds, ws, st, rows)


def test_probe_sends_an_unfilterable_chunk_to_the_dense_pass():
    # the 128K recipe (independent heads: the bound filters little) on a 1024
    # row chunk: the 128 probe rows are screened, the rest skip the pruned
    # path; the result is still the dense one bit for bit
    off, T_q, topk = 15360, 1024, 512
    x = make_prefill("chunk_128k_h32", T_q=T_q, T_k=off + T_q, q_offset=off, seed=33, with_anchor=True)
    seeds = anchor_seeds(x, topk, 2560, seed=34)
    di, ds, pi, ps, st = run_both(x, topk, seeds)
    print("bypass", st)
    assert st["bypassed_rows"] == T_q - PROBE_ROWS
    assert st["screened_pairs"] == expected_screened_pairs(off, T_q, len(seeds), st)
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))
    rows = np.array([0, 127, 128, 700, T_q - 1])
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, topk)
    check_rows(pi[rows], ps[rows], oi, osc, amax, off + rows + 1, topk, score_of, "bypass")


def test_shared_refine_stream_mixes_shared_and_own_keys():
    # groups of four rows whose queries differ: the shared stream holds only
    # the keys two or more rows keep; the result is still the dense one bit
    # for bit.  Rows 0-3 repeat query A, rows 4-7 alternate A and B, rows
    # 8-11 are four different queries built like A
    T_q, off, topk = 12, 6000, 128
    x, _ = _tight_bound_chunk("causal_16k_h64", T_q, off + T_q, off, topk, 409, 300)
    rng = np.random.default_rng(3)
    qb = x["q"][0].copy()
    qb[:14] = np.flip(qb[:14], axis=1)  # another query with the same head structure
    x["q"][5] = qb
    x["q"][7] = qb
    for t in range(8, 12):
        qt = x["q"][0].copy()
        qt[:14] = qt[:14][rng.permutation(14)][:, rng.permutation(128)]
        x["q"][t] = qt
    # seeds: every distinct query's Top-k among the keys before the chunk
    # (a tight threshold for every row), plus random keys
    top = [oracle.prefill_topk(x["q"][t:t + 1], x["w"][t:t + 1], x["k"][:off], off - 1, topk)[0][0]
           for t in (0, 5, 8, 9, 10, 11)]
    top = np.unique(np.concatenate(top))
    seeds = np.concatenate([top, random_distinct_keys(14, 0, off, 300, exclude=top)]).astype(np.int32)
    di, ds, pi, ps, st = run_both(x, topk, seeds)
    print("mixed groups", st)
    assert np.array_equal(pi, di) and np.array_equal(ps.view(np.uint32), ds.view(np.uint32))
    assert st["recovered_rows"] == 0
    check_refine_counts(st, all_refined=True)
    rows = np.arange(T_q)
    oi, osc, amax, score_of = oracle_prefill_rows(x, rows, topk)
    check_rows(pi, ps, oi, osc, amax, off + rows + 1, topk, score_of, "mixed groups")
