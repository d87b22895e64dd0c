"""Shared parity checks: CUDA Top-k lists against the fp64 oracle.

Tolerance: a GPU score may differ from the oracle's fp64 score of the same
key by at most tol = 2e-3 * max_s |I(t,s)| over the row's visible keys (fp32
tensor-core accumulation against fp64).  Where several selections are
correct (keys whose oracle scores lie within tol of the m-th score), the set
rule accepts any of them: every key the oracle scores above theta + tol must
be selected, and no selected key may score below theta - tol, where theta is
the oracle's m-th score.  Everything else is exact: row lengths, padding,
index ranges, uniqueness, and the order of the GPU list by its own fp32
scores (score descending, then smaller key).
"""

from __future__ import annotations

import numpy as np

import oracle

REL_TOL = 2e-3


def check_rows(gpu_idx, gpu_score, or_idx, or_score, or_amax, visible, topk, oracle_score_of,
               label=""):
    """Compare GPU rows with oracle rows.

    gpu_idx/gpu_score: (n, topk) numpy arrays of the GPU output rows.
    or_idx/or_score/or_amax: the oracle's rows (same order).
    visible: (n,) number of visible keys of each row.
    oracle_score_of(i, keys) -> fp64 oracle scores of `keys` in row i.
    """
    n = gpu_idx.shape[0]
    worst = 0.0
    for i in range(n):
        m = int(min(topk, visible[i]))
        gi, gs = gpu_idx[i], gpu_score[i]
        where = f"{label} row {i}"
        assert (gi[m:] == -1).all(), f"{where}: padding indices"
        assert np.isneginf(gs[m:]).all(), f"{where}: padding scores"
        if m == 0:
            continue
        sel = gi[:m].astype(np.int64)
        assert (sel >= 0).all() and (sel < visible[i]).all(), f"{where}: key outside the visible range"
        assert len(np.unique(sel)) == m, f"{where}: duplicate keys"
        s = gs[:m].astype(np.float32)
        assert np.isfinite(s).all(), f"{where}: non-finite score"
        # sorted by the GPU's own scores: descending, ties by smaller key
        bad = (s[1:] > s[:-1]) | ((s[1:] == s[:-1]) & (sel[1:] < sel[:-1]))
        assert not bad.any(), f"{where}: not sorted at {np.flatnonzero(bad)[:5]}"
        tol = REL_TOL * float(or_amax[i])
        ref = oracle_score_of(i, sel)
        err = np.abs(s.astype(np.float64) - ref)
        worst = max(worst, float(err.max() / max(or_amax[i], 1e-30)))
        assert (err <= tol).all(), f"{where}: score error {err.max():.3e} > tol {tol:.3e}"
        theta = float(or_score[i, m - 1])
        must = or_idx[i, :m][or_score[i, :m] > theta + tol]
        missing = np.setdiff1d(must, sel)
        assert missing.size == 0, f"{where}: {missing.size} keys clearly in the Top-k are missing"
        assert (ref >= theta - tol).all(), f"{where}: selected key clearly below the k-th score"
    return worst


def oracle_prefill_rows(x, rows, topk):
    """Oracle Top-k, |I| maxima and a score lookup for the listed prefill rows."""
    idx, sc, amax = oracle.prefill_topk(x["q"], x["w"], x["k"], x["q_offset"], topk, rows=rows)

    def score_of(i, keys):
        r = np.full(len(keys), rows[i], np.int64)
        return oracle.score_pairs(x["q"], x["w"], x["k"], r, keys)

    return idx, sc, amax, score_of


def oracle_decode_rows(x, topk):
    idx, sc, amax = oracle.decode_topk(x["q"], x["w"], x["k"], x["seq_len"], topk)

    def score_of(i, keys):
        return oracle.score_pairs(x["q"][i:i + 1], x["w"][i:i + 1], x["k"][i],
                                  np.zeros(len(keys), np.int64), keys)

    return idx, sc, amax, score_of
