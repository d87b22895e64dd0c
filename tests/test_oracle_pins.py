"""Pins for the CPU oracle: values and properties fixed by the pages or by
mathematics, never by the oracle itself.

Sources: "DeepSeek DSA FLOPs" (notation table, causal token-pair count, index
score equation, prefill and decode FLOP counts) and the DoSA reading notes /
163.com write-up (seed threshold, upper bound, sum-then-ReLU lower bound).
"""

import math

import numpy as np
import pytest

import oracle
from synth import bf16_bits_from_f64, bf16_bits_to_f32, make_integer_prefill, make_prefill


def _golden(path):
    out = {}
    for line in path.read_text().splitlines():
        line = line.split("#", 1)[0].strip()
        if not line:
            continue
        key, val = [x.strip() for x in line.split("=")]
        out[key] = float(val)
    return out


# ---------------------------------------------------------------- counts ----

def test_pair_counts_match_worked_numbers(golden_dir):
    g = _golden(golden_dir / "dsa_flops_worked_numbers.txt")
    T, k = g["T_128K"], g["k"]
    # the page prints N_sel at T = 131072, k = 2048
    assert oracle.n_sel(T, k) == g["N_sel_128K"]
    # N_sel for T > k also has the closed form kT - k(k-1)/2
    for T_, k_ in [(1024, 256), (5000, 2048), (2049, 2048), (10, 3)]:
        assert oracle.n_sel(T_, k_) == k_ * T_ - k_ * (k_ - 1) / 2
    # T <= k keeps every visible pair
    assert oracle.n_sel(100, 2048) == 100 * 101 / 2


def test_scoring_flops_match_worked_numbers(golden_dir):
    g = _golden(golden_dir / "dsa_flops_worked_numbers.txt")
    H, d, T = int(g["H_I"]), int(g["d_I"]), g["T_128K"]
    f = oracle.scoring_flops(oracle.n_dense(T), H, d)
    assert f == g["index_score_flops_per_T_T1"] * T * (T + 1)
    assert round(f / 1e12, 2) == g["index_score_TF_128K"]
    dec = oracle.scoring_flops(T, H, d)  # one query scanning t = T keys
    assert dec == g["decode_scan_flops_per_t"] * T
    assert round(dec / 1e9, 3) == g["decode_scan_GF_128K"]


def test_emitted_visible_pairs_and_selected_pairs():
    # count what the oracle actually emits: visible scores per row = p+1,
    # their total = T(T+1)/2, non-pad outputs = N_sel(T, k)
    T, topk = 40, 7
    x = make_integer_prefill(3, T, 2, 4)
    idx, sc, amax, full = oracle.prefill_topk(x["q"], x["w"], x["k"], 0, topk, want_scores=True)
    per_row = np.isfinite(full).sum(axis=1)
    assert (per_row == np.arange(1, T + 1)).all()
    assert per_row.sum() == T * (T + 1) // 2 == oracle.n_dense(T)
    assert (idx >= 0).sum() == oracle.n_sel(T, topk)
    # padding beyond m = min(k, p+1)
    for t in range(T):
        m = min(topk, t + 1)
        assert (idx[t, m:] == -1).all() and np.isneginf(sc[t, m:]).all()
        assert (idx[t, :m] >= 0).all() and (idx[t, :m] <= t).all()


def test_chunk_offsets_visible_counts():
    # a chunk at q_offset sees q_offset + t + 1 keys in row t
    T_k, off, T_q = 50, 30, 20
    x = make_integer_prefill(4, T_k, 1, 3, q_offset=off)
    _, _, _, full = oracle.prefill_topk(x["q"], x["w"], x["k"], off, 5, want_scores=True)
    assert (np.isfinite(full).sum(axis=1) == off + np.arange(1, T_q + 1)).all()


# ------------------------------------------------------------- scores -------

def test_hand_worked_example(golden_dir):
    lines = [l.split() for l in (golden_dir / "index_score_hand_example.txt").read_text().splitlines()
             if l.strip() and not l.startswith("#")]
    T, H, d, topk = 4, 2, 2, 2
    k = np.zeros((T, d))
    q = np.zeros((T, H, d))
    w = np.zeros((T, H), np.float32)
    I_exp, top_exp = {}, {}
    for f in lines:
        if f[0] == "k":
            k[int(f[1])] = [float(v) for v in f[2:]]
        elif f[0] == "q":
            q[int(f[1]), int(f[2])] = [float(v) for v in f[3:]]
        elif f[0] == "w":
            w[int(f[1])] = [float(v) for v in f[2:]]
        elif f[0] == "I":
            I_exp[(int(f[1]), int(f[2]))] = float(f[3])
        elif f[0] == "top":
            top_exp[int(f[1])] = [(int(f[2]), float(f[3])), (int(f[4]), float(f[5]))]
    qb, kb = bf16_bits_from_f64(q), bf16_bits_from_f64(k)
    idx, sc, amax, full = oracle.prefill_topk(qb, w, kb, 0, topk, want_scores=True)
    for (t, s), v in I_exp.items():
        assert full[t, s] == v
    for t, pairs in top_exp.items():
        for i, (ii, ss) in enumerate(pairs):
            assert idx[t, i] == ii
            assert sc[t, i] == ss or (math.isinf(ss) and np.isneginf(sc[t, i]))
    assert amax[1] == 4.0 and amax[3] == 4.0


def test_single_head_unit_weight_is_relu_dot_topk():
    # H = 1, w = 1: the index score is ReLU(q.k); the selection is a textbook
    # Top-k of that, here numpy matmul + lexsort (score desc, index asc)
    rng = np.random.default_rng(0)
    T, d, topk = 64, 16, 9
    q = bf16_bits_from_f64(rng.standard_normal((T, 1, d)))
    k = bf16_bits_from_f64(rng.standard_normal((T, d)))
    w = np.ones((T, 1), np.float32)
    idx, sc, _, full = oracle.prefill_topk(q, w, k, 0, topk, want_scores=True)
    Q = bf16_bits_to_f32(q[:, 0, :]).astype(np.float64)
    K = bf16_bits_to_f32(k).astype(np.float64)
    ref = np.maximum(Q @ K.T, 0.0)
    for t in range(T):
        np.testing.assert_allclose(full[t, :t + 1], ref[t, :t + 1], rtol=1e-13, atol=1e-13)
        order = np.lexsort((np.arange(t + 1), -ref[t, :t + 1]))[:topk]
        m = min(topk, t + 1)
        assert (idx[t, :m] == order[:m]).all()


def test_one_hot_weight_selects_one_head():
    # w = e_j isolates head j: I = ReLU(q_j . k); catches a head-stride mistake
    rng = np.random.default_rng(1)
    T, H, d = 12, 5, 8
    q = bf16_bits_from_f64(rng.standard_normal((T, H, d)))
    k = bf16_bits_from_f64(rng.standard_normal((T, d)))
    Q = bf16_bits_to_f32(q).astype(np.float64)
    K = bf16_bits_to_f32(k).astype(np.float64)
    for j in range(H):
        w = np.zeros((T, H), np.float32)
        w[:, j] = 1.0
        _, _, _, full = oracle.prefill_topk(q, w, k, 0, 3, want_scores=True)
        ref = np.maximum(Q[:, j, :] @ K.T, 0.0)
        for t in range(T):
            np.testing.assert_allclose(full[t, :t + 1], ref[t, :t + 1], rtol=1e-13, atol=1e-13)


def test_linear_in_weights_and_positively_homogeneous_in_keys():
    x = make_integer_prefill(7, 16, 3, 4)
    rng = np.random.default_rng(2)
    w1 = rng.integers(-3, 4, size=x["w"].shape).astype(np.float32)
    w2 = rng.integers(-3, 4, size=x["w"].shape).astype(np.float32)
    f = lambda w, k: oracle.prefill_topk(x["q"], w, k, 0, 4, want_scores=True)[3]
    a, b, ab = f(w1, x["k"]), f(w2, x["k"]), f(w1 + w2, x["k"])
    fin = np.isfinite(a)
    assert (a[fin] + b[fin] == ab[fin]).all()  # integers: exact in fp64
    k2 = bf16_bits_from_f64(2.0 * bf16_bits_to_f32(x["k"]).astype(np.float64))
    assert (f(w1, k2)[fin] == 2.0 * a[fin]).all()  # ReLU(2x) = 2 ReLU(x)
    kneg = bf16_bits_from_f64(-bf16_bits_to_f32(x["k"]).astype(np.float64))
    # I(k) - I(-k) = sum_j w_j (q_j . k): ReLU(x) - ReLU(-x) = x
    Q = bf16_bits_to_f32(x["q"]).astype(np.float64)
    K = bf16_bits_to_f32(x["k"]).astype(np.float64)
    lin = np.einsum("th,thd,sd->ts", w1.astype(np.float64), Q, K)
    diff = f(w1, x["k"])[fin] - f(w1, kneg)[fin]
    assert (diff == lin[fin]).all()


def test_selection_exhaustive_small():
    # every selected key outscores (or ties with a larger index than) every
    # unselected visible key; the selection is sorted; m = min(k, p+1)
    for seed in range(4):
        x = make_integer_prefill(10 + seed, 12, 3, 4, lo=-2, hi=2)
        for topk in (1, 3, 12, 20):
            idx, sc, _, full = oracle.prefill_topk(x["q"], x["w"], x["k"], 0, topk, want_scores=True)
            for t in range(12):
                m = min(topk, t + 1)
                sel = idx[t, :m]
                assert len(set(sel.tolist())) == m
                for i in range(m):
                    assert sc[t, i] == full[t, sel[i]]
                    if i:
                        assert (sc[t, i - 1] > sc[t, i]) or (sc[t, i - 1] == sc[t, i] and sel[i - 1] < sel[i])
                rest = [s for s in range(t + 1) if s not in set(sel.tolist())]
                for s in rest:
                    worst = sc[t, m - 1]
                    assert full[t, s] < worst or (full[t, s] == worst and s > sel[m - 1])


def test_decode_rows_are_last_rows_of_a_causal_prefill():
    # a decode query over a cache of length L scores keys 0..L-1; the same
    # query placed at position L-1 of a causal prefill over the same keys sees
    # the same keys.  Every sequence has its own cache.
    L = np.array([30, 17, 1, 0], np.int32)
    probs = [make_integer_prefill(21 + b, 30, 2, 4) for b in range(len(L))]
    q = np.stack([x["q"][max(l - 1, 0)] for x, l in zip(probs, L)])
    w = np.stack([x["w"][max(l - 1, 0)] for x, l in zip(probs, L)])
    kc = np.stack([x["k"] for x in probs])
    idx, sc, _ = oracle.decode_topk(q, w, kc, L, 6)
    for b, l in enumerate(L):
        if l == 0:
            assert (idx[b] == -1).all() and np.isneginf(sc[b]).all()
            continue
        pidx, psc, _ = oracle.prefill_topk(probs[b]["q"], probs[b]["w"], probs[b]["k"], 0, 6,
                                           rows=[l - 1])
        assert (idx[b] == pidx[0]).all() and (sc[b] == psc[0]).all()


# ------------------------------------------------------------- DoSA ---------

def _bf(x):
    return bf16_bits_from_f64(np.asarray(x, np.float64))


def test_sum_then_relu_lower_bound():
    # sum_j a_j ReLU(x_j) >= ReLU(sum_j a_j x_j) for a_j >= 0 (DoSA, negative heads)
    rng = np.random.default_rng(5)
    for _ in range(200):
        a = np.abs(rng.standard_normal(7))
        x = rng.standard_normal(7) * 3
        assert (a * np.maximum(x, 0)).sum() >= max((a * x).sum(), 0.0) - 1e-12


def test_bound_is_exact_for_a_single_negative_omitted_head():
    # retained heads = all positive heads, one negative head omitted: the folded
    # negative term is that head's exact penalty, so U == I.  A wrong sign or a
    # dropped term in the negative fold breaks this equality.
    d = 4
    q = _bf([[1, 0.5, 0, 0], [0, 1, -1, 0], [0.5, 0, 1, 1]])
    w = np.array([1.0, 2.0, -1.5], np.float32)
    # keys 0-1 are the planner's sample (they make heads 0 and 1 the important
    # ones); keys 2-6 are scored
    keys = _bf([[0, 4, -4, 0], [4, 0, 0, 0],
                [1, 1, 0, 0], [0, 0, 1, 1], [1, -1, 1, 0], [2, 0, 0, 1], [0, 1, 1, 0]])
    plan = oracle.dosa_plan(q, w, keys, np.arange(2, dtype=np.int32), r=2)
    assert sorted(np.flatnonzero(plan["role"] == 0).tolist()) == [0, 1]
    assert plan["role"][2] == 2
    for s in range(2, 7):
        I = oracle.row_scores(q, w, keys[s:s + 1], 1)[0]
        U = oracle.dosa_bound(plan, q, w, keys[s])
        assert abs(U - I) < 1e-12, (s, U, I)


def test_bound_is_exact_when_positive_heads_lie_in_the_retained_span():
    # q_2 = 2 q_0 - 3 q_1 (a positive omitted head in the span of the retained
    # heads): residual 0, c = (2, -3), alpha = w_2 * (2, 3).  The bound
    # (w x + w (|c_0 d_0| + |c_1 d_1|)) / 2 equals w ReLU(x) exactly when the
    # two terms c_i d_i share a sign, and is strictly above it otherwise.
    q = _bf([[1, 0, 2, 0], [0, 1, 0, 1], [2, -3, 4, -3]])
    w = np.array([3.0, 2.0, 0.5], np.float32)
    keys = _bf([[1, 2, 0, 1], [-1, 0, 1, 0], [0, 0, 0, 1], [1, 1, 1, 1], [3, 0, -1, 2],
                [1, -1, 0, -1]])
    plan = oracle.dosa_plan(q, w, keys, np.arange(6, dtype=np.int32), r=2)
    assert sorted(np.flatnonzero(plan["role"] == 0).tolist()) == [0, 1]
    np.testing.assert_allclose(plan["alpha"][:2], [0.5 * 2, 0.5 * 3], atol=1e-12)
    assert abs(plan["beta"]) < 1e-12
    np.testing.assert_allclose(plan["q_pos"], 0.5 * np.array([2, -3, 4, -3]), atol=1e-15)
    # by hand, d = (q_0.k, q_1.k), x = q_2.k:
    #  k1: d=(1,0) x=2   I=3+0+1=4   U=3+0.5+0.5=4
    #  k2: d=(0,1) x=-3  I=0+2+0=2   U=2-0.75+0.75=2
    #  k5: d=(1,-2) x=8  I=3+0+4=7   U=3+2+2=7
    #  k0: d=(1,3) x=-7  I=3+6+0=9   U=9-1.75+2.75=10
    #  k3: d=(3,2) x=0   I=9+4+0=13  U=13+0+3=16
    #  k4: d=(1,2) x=-4  I=3+4+0=7   U=7-1+2=8
    tight = {1: 4.0, 2: 2.0, 5: 7.0}
    loose = {0: (9.0, 10.0), 3: (13.0, 16.0), 4: (7.0, 8.0)}
    for s in range(6):
        I = oracle.row_scores(q, w, keys[s:s + 1], 1)[0]
        U = oracle.dosa_bound(plan, q, w, keys[s])
        if s in tight:
            assert I == tight[s] and abs(U - I) < 1e-12, (s, U, I)
        else:
            assert I == loose[s][0] and abs(U - loose[s][1]) < 1e-12, (s, U, I)


def test_bound_is_exact_for_keys_along_the_residual():
    # orthogonal positive omitted head: c = 0, rho = ||q_j||; for keys parallel
    # or antiparallel to q_j the Cauchy-Schwarz term is attained and U == I.
    q = _bf([[1, 0], [0, 2]])
    w = np.array([4.0, 1.5], np.float32)
    samples = _bf([[1, 0], [1, 0]])
    plan = oracle.dosa_plan(q, w, samples, np.arange(2, dtype=np.int32), r=1)
    assert plan["role"][0] == 0 and plan["role"][1] == 1
    assert abs(plan["beta"] - 1.5 * 2.0) < 1e-12  # w_1 * ||q_1||
    for key in ([0, 1], [0, -1], [0, 3], [0, -2]):
        ks = _bf([key])[0]
        I = oracle.row_scores(q, w, ks[None], 1)[0]
        U = oracle.dosa_bound(plan, q, w, ks)
        assert abs(U - I) < 1e-12
    # and strictly above I off that line
    ks = _bf([[1, 1]])[0]
    assert oracle.dosa_bound(plan, q, w, ks) > oracle.row_scores(q, w, ks[None], 1)[0] + 1e-6


def test_all_heads_retained_gives_the_exact_score():
    x = make_prefill("causal_1k_h64", T_q=4, T_k=300)
    q, w, k = x["q"][2], x["w"][2], x["k"]
    plan = oracle.dosa_plan(q, w, k, np.arange(0, 256, 2, dtype=np.int32), r=64)
    I = oracle.row_scores(q, w, k, 300)
    U = np.array([oracle.dosa_bound(plan, q, w, k[s]) for s in range(300)])
    assert (U == I).all()


@pytest.mark.parametrize("recipe,r,sign", [
    ("causal_1k_h64", 14, None), ("causal_1k_h64", 1, None), ("causal_1k_h64", 63, None),
    ("causal_16k_h64", 14, None), ("causal_1k_h64", 14, "neg"), ("causal_1k_h64", 14, "pos"),
])
def test_dosa_row_is_lossless_and_the_bound_is_safe(recipe, r, sign):
    # U >= I on every screened key, tau <= the true k-th score, and the pruned
    # selection equals the dense one exactly (DoSA keeps the original Top-k).
    T, off, topk, n_seed = 700, 400, 64, 160
    x = make_prefill(recipe, T_q=T - off, T_k=T, q_offset=off)
    rng = np.random.default_rng(9)
    seeds = rng.choice(off, size=n_seed, replace=False).astype(np.int32)
    for t in (0, 150, T - off - 1):
        w = x["w"][t].copy()
        if sign == "neg":
            w = -np.abs(w)
        elif sign == "pos":
            w = np.abs(w)
        p = off + t
        res = oracle.dosa_row(x["q"][t], w, x["k"], p, seeds, topk, r)
        dense_idx, dense_sc, _ = oracle.prefill_topk(x["q"][t:t + 1], w[None], x["k"][:p + 1],
                                                     p, topk)
        assert res["min_gap"] >= -1e-9 * (1 + abs(res["tau"]))
        assert res["tau"] <= dense_sc[0, topk - 1]
        assert (res["idx"] == dense_idx[0]).all()
        assert (res["score"] == dense_sc[0]).all()
        assert res["screened"] == p + 1 - n_seed
        assert res["survivors"] <= res["screened"]


def test_planner_sample_positions():
    # "DoSA" reading notes, annotation ADQKPC5Q, step 1: the planner samples
    # 128 positions 32 + 64 i of the seed region (12,288 seeds)
    seeds = np.arange(12288, dtype=np.int32) * 3
    s = oracle.dosa_sample(seeds)
    assert s.tolist() == [3 * (32 + 64 * i) for i in range(128)]
    # shorter lists keep the even spacing: every entry when there are at most 128
    assert oracle.dosa_sample(seeds[:5]).tolist() == [0, 3, 6, 9, 12]
    assert oracle.dosa_sample(seeds[:1024]).tolist() == [3 * (4 + 8 * i) for i in range(128)]


# ------------------------------------------------------- pair scorer ------

def test_score_pairs_matches_a_numpy_matmul_at_random_pairs():
    # the per-pair scorer every GPU parity test uses: I(t, s) from the widened
    # bf16/fp32 inputs by numpy (einsum + ReLU + weighted sum), at random
    # (row, key) pairs, for a chunk layout (rows index q/w, keys index k) and
    # for one decode sequence's cache
    rng = np.random.default_rng(17)
    for H, d in ((64, 128), (32, 128), (3, 8)):
        T_q, T_k = 9, 300
        q = bf16_bits_from_f64(rng.standard_normal((T_q, H, d)) / 4)
        k = bf16_bits_from_f64(rng.standard_normal((T_k, d)))
        w = rng.standard_normal((T_q, H)).astype(np.float32)
        rows = rng.integers(0, T_q, size=200)
        keys = rng.integers(0, T_k, size=200)
        got = oracle.score_pairs(q, w, k, rows, keys)
        Q = bf16_bits_to_f32(q).astype(np.float64)
        K = bf16_bits_to_f32(k).astype(np.float64)
        dots = np.einsum("nhd,nd->nh", Q[rows], K[keys])
        ref = (w[rows].astype(np.float64) * np.maximum(dots, 0.0)).sum(axis=1)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    # a wrong row or key stride would pick another vector: distinct rows and
    # keys give distinct scores here, and swapping the two index lists changes
    # the result
    assert not np.allclose(oracle.score_pairs(q, w, k, rows, keys),
                           oracle.score_pairs(q, w, k, rows[::-1], keys))


def test_score_pairs_agrees_with_the_chunk_and_decode_scores():
    # the same pairs scored through the chunked prefill (q_offset > 0) and the
    # batched decode layouts give identical values
    x = make_prefill("chunk_128k_h32", T_q=6, T_k=500, q_offset=494)
    _, _, _, full = oracle.prefill_topk(x["q"], x["w"], x["k"], 494, 4, want_scores=True)
    rng = np.random.default_rng(3)
    rows = rng.integers(0, 6, size=50)
    keys = np.array([rng.integers(0, 494 + r + 1) for r in rows])
    got = oracle.score_pairs(x["q"], x["w"], x["k"], rows, keys)
    assert (got == full[rows, keys]).all()
    # decode: sequence b's query against its own cache
    L = np.array([500, 300], np.int32)
    kc = np.stack([x["k"], x["k"][::-1].copy()])
    q, w = x["q"][:2], x["w"][:2]
    idx, sc, _ = oracle.decode_topk(q, w, kc, L, 5)
    for b in range(2):
        got = oracle.score_pairs(q[b:b + 1], w[b:b + 1], kc[b], np.zeros(5, np.int64), idx[b])
        assert (got == sc[b]).all()


# ------------------------------------------------------------------ FP8 ----

def test_e4m3_decode_matches_torch_float8():
    # every FP8 E4M3 code decodes to the value a library routine gives
    # (torch.float8_e4m3fn), NaN codes included
    import torch
    codes = np.arange(256, dtype=np.uint8)
    got = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().double().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert (got[~np.isnan(got)] == ref[~np.isnan(ref)]).all()
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x38] == 1.0


def test_fp8_scores_with_unit_scales_equal_the_bf16_scores():
    # every E4M3 value is exactly a bf16 value, so with unit scales the FP8
    # definition is the bf16 one on the same numbers
    from synth import quantize_e4m3_rows
    x = make_prefill("causal_16k_h64", T_q=12, T_k=300, q_offset=288, seed=5)
    q8, _ = quantize_e4m3_rows(x["q"])
    k8, _ = quantize_e4m3_rows(x["k"])
    qb = bf16_bits_from_f64(oracle.e4m3_decode(q8).reshape(q8.shape))
    kb = bf16_bits_from_f64(oracle.e4m3_decode(k8).reshape(k8.shape))
    ones_q, ones_k = np.ones(q8.shape[:2], np.float32), np.ones(k8.shape[0], np.float32)
    fi, fs, fa = oracle.prefill_topk_fp8(q8, ones_q, x["w"], k8, ones_k, 288, 40)
    bi, bs, ba = oracle.prefill_topk(qb, x["w"], kb, 288, 40)
    assert (fi == bi).all() and (fs == bs).all() and (fa == ba).all()


def test_fp8_scales_act_as_positive_factors():
    # a key scale multiplies every score of that key; a query head scale
    # multiplies that head's weight (ReLU is positively homogeneous)
    from synth import make_prefill_fp8
    x = make_prefill_fp8("causal_16k_h64", T_q=4, T_k=64, q_offset=60, seed=6)
    rows = np.repeat(np.arange(4), 64)
    keys = np.tile(np.arange(64), 4)
    base = oracle.score_pairs_fp8(x["q8"], x["q_scale"], x["w"], x["k8"], x["k_scale"], rows, keys)
    ks2 = x["k_scale"] * np.float32(2.0)
    assert np.allclose(oracle.score_pairs_fp8(x["q8"], x["q_scale"], x["w"], x["k8"], ks2, rows, keys),
                       2.0 * base, rtol=1e-13, atol=0)
    qs3, w3 = x["q_scale"].copy(), x["w"].copy()
    qs3[:, 5] *= np.float32(4.0)
    w3[:, 5] *= np.float32(4.0)
    a = oracle.score_pairs_fp8(x["q8"], qs3, x["w"], x["k8"], x["k_scale"], rows, keys)
    b = oracle.score_pairs_fp8(x["q8"], x["q_scale"], w3, x["k8"], x["k_scale"], rows, keys)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-300)


# ------------------------------------------------------- history seeds ----

def test_seeds_from_history_hand_example():
    # 163.com write-up, section 03: seeds by historical selection frequency.
    # Rows selected keys {5,2,7}, {2,7,-1}, {7,9,2}, {0,5,7}: counts
    # 7:4, 2:3, 5:2, 0:1, 9:1, others 0; ties by the smaller key
    prev = np.array([[5, 2, 7], [2, 7, -1], [7, 9, 2], [0, 5, 7]], np.int32)
    # -> the seven most selected: 7, 2, 5, then 0 and 9 (count 1), then the
    # never-selected 1 and 3; listed in ascending key order
    seeds, counts = oracle.seeds_from_history(prev, 10, 7)
    assert seeds.tolist() == [0, 1, 2, 3, 5, 7, 9]
    assert counts.tolist() == [1, 0, 3, 0, 0, 2, 0, 4, 0, 1]
    # keys at or beyond n_keys (not visible to the next chunk) never count
    seeds, counts = oracle.seeds_from_history(prev, 6, 3)
    assert seeds.tolist() == [0, 2, 5] and counts.tolist() == [1, 0, 3, 0, 0, 2]


def test_seeds_from_history_properties():
    # every chosen key was selected at least as often as every key left out,
    # the seeds are distinct, and counts add up to the valid entries
    rng = np.random.default_rng(4)
    prev = rng.integers(-1, 400, size=(50, 16)).astype(np.int32)
    seeds, counts = oracle.seeds_from_history(prev, 300, 64)
    assert len(set(seeds.tolist())) == 64 and (seeds >= 0).all() and (seeds < 300).all()
    out = np.setdiff1d(np.arange(300), seeds)
    assert counts[seeds].min() >= counts[out].max()
    assert counts.sum() == ((prev >= 0) & (prev < 300)).sum()
