"""CPU oracle for the lightning-indexer hot path (fp64, plain C + OpenMP).

TEST INFRASTRUCTURE ONLY: tests, the smoke check and the benchmark's CPU
baseline leg may import this package; the product path never does.  It shares
no code with the CUDA library.  The C source cites the passages it follows.

Functions take numpy arrays: q/k as bf16 bit patterns (uint16), w as float32.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "dsa_oracle.c"
_LIB = _HERE / "liboracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile the oracle with gcc (-O2, OpenMP) next to its source."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(f".{os.getpid()}.tmp")
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", str(tmp), str(_SRC), "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(str(build()))
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        I32 = ctypes.c_int
        D = ctypes.c_double
        _lib.oracle_row_scores.argtypes = [P, P, P, I64, I32, I32, P]
        _lib.oracle_score_pairs.argtypes = [P, P, P, I32, I32, I64, P, P, P, I32]
        _lib.oracle_prefill_topk.argtypes = [P, P, P, I64, I64, I64, I32, I32, I32, P, I64,
                                             P, P, P, P, I32]
        _lib.oracle_prefill_topk.restype = I32
        _lib.oracle_decode_topk.argtypes = [P, P, P, P, I64, I64, I32, I32, I32, P, P, P, I32]
        _lib.oracle_decode_topk.restype = I32
        _lib.oracle_dosa_plan_size.argtypes = [I32, I32]
        _lib.oracle_dosa_plan_size.restype = I32
        _lib.oracle_dosa_plan.argtypes = [P, P, P, P, I32, I32, I32, I32, P]
        _lib.oracle_dosa_plan.restype = I32
        _lib.oracle_dosa_bound.argtypes = [P, P, P, P, I32, I32]
        _lib.oracle_dosa_bound.restype = D
        _lib.oracle_dosa_sample.argtypes = [P, I32, P]
        _lib.oracle_dosa_sample.restype = I32
        _lib.oracle_dosa_row.argtypes = [P, P, P, I64, P, I32, I32, I32, I32, I32, P, P, P, P,
                                         P, P]
        _lib.oracle_dosa_row.restype = I32
        U8 = P
        _lib.oracle_e4m3_decode.argtypes = [U8, I64, P]
        _lib.oracle_prefill_topk_fp8.argtypes = [P, P, P, P, P, I64, I64, I64, I32, I32, I32, P, I64,
                                                 P, P, P, I32]
        _lib.oracle_prefill_topk_fp8.restype = I32
        _lib.oracle_score_pairs_fp8.argtypes = [P, P, P, P, P, I32, I32, I64, P, P, P, I32]
        _lib.oracle_seeds_from_history.argtypes = [P, I64, I32, I64, I32, P, P]
        _lib.oracle_seeds_from_history.restype = I32
        for f in ("oracle_n_dense",):
            getattr(_lib, f).argtypes = [D]
            getattr(_lib, f).restype = D
        _lib.oracle_n_sel.argtypes = [D, D]
        _lib.oracle_n_sel.restype = D
        _lib.oracle_scoring_flops.argtypes = [D, I32, I32]
        _lib.oracle_scoring_flops.restype = D
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def threads() -> int:
    """Host threads the oracle uses: every core this process may run on."""
    return len(os.sched_getaffinity(0))


def row_scores(q_row, w_row, k, n_keys: int) -> np.ndarray:
    """I(t, s) for s < n_keys, one query row q_row (H, d)."""
    q_row, w_row, k = _c(q_row, np.uint16), _c(w_row, np.float32), _c(k, np.uint16)
    H, d = q_row.shape
    out = np.empty(n_keys, np.float64)
    _load().oracle_row_scores(_p(q_row), _p(w_row), _p(k), n_keys, H, d, _p(out))
    return out


def score_pairs(q, w, k, q_rows, keys, n_threads: int | None = None) -> np.ndarray:
    """I for arbitrary pairs: q_rows index the first axis of q/w, keys index k."""
    q, w, k = _c(q, np.uint16), _c(w, np.float32), _c(k, np.uint16)
    q_rows, keys = _c(q_rows, np.int64).ravel(), _c(keys, np.int64).ravel()
    H, d = q.shape[-2], q.shape[-1]
    out = np.empty(q_rows.shape[0], np.float64)
    _load().oracle_score_pairs(_p(q), _p(w), _p(k), H, d, q_rows.shape[0], _p(q_rows),
                               _p(keys), _p(out), n_threads or threads())
    return out


def prefill_topk(q, w, k, q_offset: int, topk: int, rows=None, want_scores: bool = False,
                 n_threads: int | None = None):
    """Sorted Top-m per listed row of a chunked causal prefill.

    Returns (idx (n,topk) int32, score (n,topk) f64, absmax (n,) f64[, scores (n,T_k)]).
    """
    q, w, k = _c(q, np.uint16), _c(w, np.float32), _c(k, np.uint16)
    T_q, H, d = q.shape
    T_k = k.shape[0]
    rows = np.arange(T_q, dtype=np.int64) if rows is None else _c(rows, np.int64)
    n = rows.shape[0]
    idx = np.empty((n, topk), np.int32)
    sc = np.empty((n, topk), np.float64)
    amax = np.empty(n, np.float64)
    full = np.empty((n, T_k), np.float64) if want_scores else None
    rc = _load().oracle_prefill_topk(_p(q), _p(w), _p(k), q_offset, T_q, T_k, H, d, topk,
                                     _p(rows), n, _p(idx), _p(sc), _p(amax),
                                     _p(full) if want_scores else None, n_threads or threads())
    if rc != 0:
        raise ValueError("oracle_prefill_topk: bad arguments")
    return (idx, sc, amax, full) if want_scores else (idx, sc, amax)


def decode_topk(q, w, k, seq_len, topk: int, n_threads: int | None = None):
    """Sorted Top-m per sequence of a batched decode step."""
    q, w, k = _c(q, np.uint16), _c(w, np.float32), _c(k, np.uint16)
    seq_len = _c(seq_len, np.int32)
    B, H, d = q.shape
    t_cap = k.shape[1]
    idx = np.empty((B, topk), np.int32)
    sc = np.empty((B, topk), np.float64)
    amax = np.empty(B, np.float64)
    rc = _load().oracle_decode_topk(_p(q), _p(w), _p(k), _p(seq_len), B, t_cap, H, d, topk,
                                    _p(idx), _p(sc), _p(amax), n_threads or threads())
    if rc != 0:
        raise ValueError("oracle_decode_topk: bad arguments")
    return idx, sc, amax


def e4m3_decode(codes) -> np.ndarray:
    """Values of FP8 E4M3 codes (uint8), in fp64."""
    codes = _c(codes, np.uint8).ravel()
    out = np.empty(codes.shape[0], np.float64)
    _load().oracle_e4m3_decode(_p(codes), codes.shape[0], _p(out))
    return out


def prefill_topk_fp8(q, q_scale, w, k, k_scale, q_offset: int, topk: int, rows=None,
                     n_threads: int | None = None):
    """prefill_topk on FP8 inputs: q (T_q,H,d) / k (T_k,d) E4M3 codes with fp32
    scales q_scale (T_q,H) and k_scale (T_k,).  Returns (idx, score, absmax)."""
    q, k = _c(q, np.uint8), _c(k, np.uint8)
    q_scale, w, k_scale = _c(q_scale, np.float32), _c(w, np.float32), _c(k_scale, np.float32)
    T_q, H, d = q.shape
    T_k = k.shape[0]
    rows = np.arange(T_q, dtype=np.int64) if rows is None else _c(rows, np.int64)
    n = rows.shape[0]
    idx = np.empty((n, topk), np.int32)
    sc = np.empty((n, topk), np.float64)
    amax = np.empty(n, np.float64)
    rc = _load().oracle_prefill_topk_fp8(_p(q), _p(q_scale), _p(w), _p(k), _p(k_scale), q_offset, T_q,
                                         T_k, H, d, topk, _p(rows), n, _p(idx), _p(sc), _p(amax),
                                         n_threads or threads())
    if rc != 0:
        raise ValueError("oracle_prefill_topk_fp8: bad arguments")
    return idx, sc, amax


def score_pairs_fp8(q, q_scale, w, k, k_scale, q_rows, keys, n_threads: int | None = None) -> np.ndarray:
    q, k = _c(q, np.uint8), _c(k, np.uint8)
    q_scale, w, k_scale = _c(q_scale, np.float32), _c(w, np.float32), _c(k_scale, np.float32)
    q_rows, keys = _c(q_rows, np.int64).ravel(), _c(keys, np.int64).ravel()
    H, d = q.shape[-2], q.shape[-1]
    out = np.empty(q_rows.shape[0], np.float64)
    _load().oracle_score_pairs_fp8(_p(q), _p(q_scale), _p(w), _p(k), _p(k_scale), H, d, q_rows.shape[0],
                                   _p(q_rows), _p(keys), _p(out), n_threads or threads())
    return out


def seeds_from_history(prev_idx, n_keys: int, n_seed: int):
    """The n_seed keys below n_keys most often selected in prev_idx (rows of
    earlier Top-k lists, -1 padding ignored), ties by the smaller key; returns
    (seeds int32 in ascending key order, counts (n_keys,) int64)."""
    prev = _c(prev_idx, np.int32)
    n_rows, topk = prev.shape
    seeds = np.empty(n_seed, np.int32)
    counts = np.empty(n_keys, np.int64)
    rc = _load().oracle_seeds_from_history(_p(prev), n_rows, topk, n_keys, n_seed, _p(seeds), _p(counts))
    if rc != 0:
        raise ValueError("oracle_seeds_from_history: bad arguments")
    return seeds, counts


def dosa_sample(seeds) -> np.ndarray:
    seeds = _c(seeds, np.int32)
    out = np.empty(128, np.int32)
    m = _load().oracle_dosa_sample(_p(seeds), seeds.shape[0], _p(out))
    return out[:m].copy()


def dosa_plan(q_row, w_row, k, sample_keys, r: int) -> dict:
    """The fp64 screening plan of one query row (see the C source)."""
    q_row, w_row, k = _c(q_row, np.uint16), _c(w_row, np.float32), _c(k, np.uint16)
    sample_keys = _c(sample_keys, np.int32)
    H, d = q_row.shape
    plan = np.empty(_load().oracle_dosa_plan_size(H, d), np.float64)
    rc = _lib.oracle_dosa_plan(_p(q_row), _p(w_row), _p(k), _p(sample_keys),
                               sample_keys.shape[0], H, d, r, _p(plan))
    if rc != 0:
        raise ValueError("oracle_dosa_plan: bad arguments")
    return dict(raw=plan, role=plan[1:1 + H].astype(int), alpha=plan[1 + H:1 + 2 * H],
                beta=plan[1 + 2 * H], q_pos=plan[2 + 2 * H:2 + 2 * H + d],
                q_neg=plan[2 + 2 * H + d:2 + 2 * H + 2 * d])


def dosa_bound(plan: dict, q_row, w_row, k_s) -> float:
    q_row, w_row, k_s = _c(q_row, np.uint16), _c(w_row, np.float32), _c(k_s, np.uint16)
    H, d = q_row.shape
    return _load().oracle_dosa_bound(_p(plan["raw"]), _p(q_row), _p(w_row), _p(k_s), H, d)


def dosa_row(q_row, w_row, k, p: int, seeds, topk: int, r: int, want_U: bool = False) -> dict:
    """Pruned selection of one row at position p, with its checks."""
    q_row, w_row, k = _c(q_row, np.uint16), _c(w_row, np.float32), _c(k, np.uint16)
    seeds = _c(seeds, np.int32)
    H, d = q_row.shape
    idx = np.empty(topk, np.int32)
    sc = np.empty(topk, np.float64)
    tau = np.zeros(1, np.float64)
    stats = np.zeros(3, np.int64)
    gap = np.zeros(1, np.float64)
    U = np.empty(p + 1, np.float64) if want_U else None
    rc = _load().oracle_dosa_row(_p(q_row), _p(w_row), _p(k), p, _p(seeds), seeds.shape[0],
                                 topk, r, H, d, _p(idx), _p(sc), _p(tau), _p(stats), _p(gap),
                                 _p(U) if want_U else None)
    if rc != 0:
        raise ValueError(f"oracle_dosa_row: status {rc}")
    return dict(idx=idx, score=sc, tau=float(tau[0]), screened=int(stats[0]),
                survivors=int(stats[1]), records=int(stats[2]), min_gap=float(gap[0]), U=U)


def n_dense(T: float) -> float:
    return _load().oracle_n_dense(float(T))


def n_sel(T: float, k: float) -> float:
    return _load().oracle_n_sel(float(T), float(k))


def scoring_flops(pairs: float, H: int, d: int) -> float:
    return _load().oracle_scoring_flops(float(pairs), H, d)
