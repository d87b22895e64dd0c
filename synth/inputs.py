"""Seeded synthetic workloads shaped like the DeepSeek-V3.2 lightning indexer.

Shapes follow the notation table of "DeepSeek DSA FLOPs" (Notation): H^I index
heads of width d^I = 128 share one key vector per position; queries carry H^I
rows, head weights w are fp32.  q and k are stored as raw bf16 bit patterns
(uint16) produced by round-to-nearest-even from fp64 draws; w stays fp32.

Value recipes (the pages fix none; these are the stated stand-ins for model
activations, which are not available here):

* ``gauss``   q, k ~ N(0,1)/sqrt(128); w ~ N(0, 1/8).
* ``lowrank`` k_s = U z_s + 0.3 e_s with U a d x r matrix of N(0, 1/r) entries,
  z_s ~ N(0, I_r), e_s ~ N(0, I_d).  Every query head row is drawn the same way
  from the same U.  w ~ N(0, 1/8).
* ``domains`` keys in three contiguous thirds, each third from its own basis
  of rank 8 / 16 / 32; queries from the last third's basis; w has magnitude
  |N(0, 1/8)| and is negative with probability 0.4.

``head_rank`` > 0 (any key recipe): a row's H query heads are no longer
independent draws; they are mixtures of ``head_rank`` per-row latent vectors,
q_{t,j} = sum_m A_{j,m} b_{t,m} + 0.05 e_{t,j}, with one mixing matrix
A ~ N(0, 1/head_rank) (H x head_rank) for the whole input and b_{t,m}
drawn like a query row of the key recipe.  It stands in for index heads that
are projections of one shared query latent.

Nothing here computes an index score or selects keys.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

BASE_SEED = 20261202
_CHUNK_ROWS = 1 << 16


@dataclass(frozen=True)
class Workload:
    """One named input configuration (sizes, value recipe, RNG seed)."""

    name: str
    kind: str  # "prefill" | "decode"
    H: int
    d: int
    topk: int
    keys: str  # "gauss" | "lowrank" | "domains"
    seed: int
    T_q: int = 0
    T_k: int = 0
    q_offset: int = 0
    B: int = 0
    t_cap: int = 0
    rank: int = 16
    n_seed: int = 0  # DoSA seed-set size (0: no seed set)
    n_anchor: int = 0  # seeds taken from an anchor query's selection
    head_rank: int = 0  # > 0: heads are mixtures of head_rank latent rows
    notes: str = field(default="", compare=False)

    @property
    def visible_pairs(self) -> int:
        """Causally visible (query, key) pairs: sum over rows of (p_t + 1)."""
        if self.kind == "decode":
            return self.B * self.t_cap
        a = self.q_offset + 1
        b = self.q_offset + self.T_q
        return (a + b) * self.T_q // 2


WORKLOADS = {
    w.name: w
    for w in [
        Workload("causal_1k_h64", "prefill", H=64, d=128, topk=256, keys="gauss",
                 seed=BASE_SEED + 1, T_q=1024, T_k=1024, q_offset=0,
                 notes="tiny full-causal prefill, oracle-sized"),
        Workload("causal_16k_h64", "prefill", H=64, d=128, topk=2048, keys="lowrank",
                 seed=BASE_SEED + 2, T_q=16384, T_k=16384, q_offset=0, rank=16,
                 notes="dense causal prefill at the DeepSeek-V3.2 indexer shape"),
        Workload("chunk_128k_h32", "prefill", H=32, d=128, topk=2048, keys="lowrank",
                 seed=BASE_SEED + 3, T_q=8192, T_k=131072, q_offset=122880, rank=16,
                 n_seed=12288, n_anchor=2048,
                 notes="8192-row chunk at the end of a 128K context"),
        Workload("chunk_1m_h64", "prefill", H=64, d=128, topk=2048, keys="domains",
                 seed=BASE_SEED + 4, T_q=4096, T_k=1048576, q_offset=1044480,
                 n_seed=12288, n_anchor=2048,
                 notes="4096-row chunk at the end of a 1M context, three key domains"),
        Workload("decode_64x128k_h64", "decode", H=64, d=128, topk=2048, keys="lowrank",
                 seed=BASE_SEED + 5, B=64, t_cap=131072, rank=16,
                 notes="64 sequences, one new query each, 128K-key caches"),
    ]
}


# --------------------------------------------------------------------------
# bf16 bit patterns
# --------------------------------------------------------------------------

def bf16_bits_from_f64(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to bf16 (round to nearest, ties to even), return bits.

    The rounding is done once, directly from fp64 (no fp32 intermediate, so no
    double rounding).  Inputs must be finite and inside the normal bf16 range
    (|x| < 3e38 and either 0 or |x| > 1.2e-38); the recipes here never leave it.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    drop = np.uint64(45)  # 52 fp64 mantissa bits - 7 bf16 mantissa bits
    half = np.uint64((1 << 44) - 1)
    lsb = (bits >> drop) & np.uint64(1)
    rounded = (bits + half + lsb) & ~np.uint64((1 << 45) - 1)
    as_f32 = rounded.view(np.float64).astype(np.float32)  # exact: 8 significant bits
    return (as_f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 values."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# recipes
# --------------------------------------------------------------------------

def _basis(rng: np.random.Generator, d: int, r: int) -> np.ndarray:
    return rng.standard_normal((d, r)) / np.sqrt(r)


def _lowrank_rows(rng: np.random.Generator, U: np.ndarray, n: int, noise: float,
                  out: np.ndarray) -> None:
    """Fill ``out`` (n, d) uint16 with bf16(U z + noise * e), chunked."""
    d, r = U.shape
    for s in range(0, n, _CHUNK_ROWS):
        m = min(_CHUNK_ROWS, n - s)
        z = rng.standard_normal((m, r))
        e = rng.standard_normal((m, d))
        out[s:s + m] = bf16_bits_from_f64(z @ U.T + noise * e)


def _gauss_rows(rng: np.random.Generator, n: int, d: int, scale: float,
                out: np.ndarray) -> None:
    for s in range(0, n, _CHUNK_ROWS):
        m = min(_CHUNK_ROWS, n - s)
        out[s:s + m] = bf16_bits_from_f64(rng.standard_normal((m, d)) * scale)


def _weights(rng: np.random.Generator, shape, recipe: str) -> np.ndarray:
    sd = np.sqrt(1.0 / 8.0)
    if recipe == "domains":
        mag = np.abs(rng.standard_normal(shape)) * sd
        neg = rng.random(shape) < 0.4
        return np.where(neg, -mag, mag).astype(np.float32)
    return (rng.standard_normal(shape) * sd).astype(np.float32)


def _mix_heads(rng: np.random.Generator, latent: np.ndarray, A: np.ndarray,
               out: np.ndarray) -> None:
    """out (rows*H, d) <- bf16 of per-row mixtures A @ latent of the latent rows (rows*r, d)."""
    H, r = A.shape
    d = latent.shape[1]
    rows = latent.shape[0] // r
    lat = bf16_bits_to_f32(latent).astype(np.float64).reshape(rows, r, d)
    for s in range(0, rows, 4096):
        e = min(rows, s + 4096)
        mix = np.einsum("hm,tmd->thd", A, lat[s:e])
        noise = 0.05 * rng.standard_normal(mix.shape)
        out[s * H:e * H] = bf16_bits_from_f64(mix + noise).reshape(-1, d)


def make_prefill(wl: Workload | str, *, T_q: int | None = None, T_k: int | None = None,
                 q_offset: int | None = None, seed: int | None = None,
                 with_anchor: bool = False, head_rank: int | None = None) -> dict:
    """Generate q (T_q,H,d) bf16 bits, w (T_q,H) fp32 and k (T_k,d) bf16 bits.

    The size overrides make smaller cases of the same recipe.  With
    ``with_anchor`` one extra query row (the row at position q_offset-1, just
    before the chunk) is drawn after the chunk's rows; it is returned as
    ``q_anchor`` (H,d) / ``w_anchor`` (H,).
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    T_q = wl.T_q if T_q is None else T_q
    T_k = wl.T_k if T_k is None else T_k
    q_offset = wl.q_offset if q_offset is None else q_offset
    if not (0 <= q_offset and q_offset + T_q <= T_k):
        raise ValueError("need 0 <= q_offset and q_offset + T_q <= T_k")
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    H, d = wl.H, wl.d
    k = np.empty((T_k, d), np.uint16)
    q = np.empty((T_q * H, d), np.uint16)
    out = {}
    if wl.keys == "gauss":
        _gauss_rows(rng, T_k, d, 1.0 / np.sqrt(128.0), k)
        _gauss_rows(rng, T_q * H, d, 1.0 / np.sqrt(128.0), q)
        w = _weights(rng, (T_q, H), "gauss")
        if with_anchor:
            qa = np.empty((H, d), np.uint16)
            _gauss_rows(rng, H, d, 1.0 / np.sqrt(128.0), qa)
            out.update(q_anchor=qa, w_anchor=_weights(rng, (H,), "gauss"))
    elif wl.keys == "lowrank":
        U = _basis(rng, d, wl.rank)
        _lowrank_rows(rng, U, T_k, 0.3, k)
        _lowrank_rows(rng, U, T_q * H, 0.3, q)
        w = _weights(rng, (T_q, H), "lowrank")
        if with_anchor:
            qa = np.empty((H, d), np.uint16)
            _lowrank_rows(rng, U, H, 0.3, qa)
            out.update(q_anchor=qa, w_anchor=_weights(rng, (H,), "lowrank"))
    elif wl.keys == "domains":
        bases = [_basis(rng, d, r) for r in (8, 16, 32)]
        edges = [0, T_k // 3, 2 * T_k // 3, T_k]
        for i in range(3):
            _lowrank_rows(rng, bases[i], edges[i + 1] - edges[i], 0.3, k[edges[i]:edges[i + 1]])
        _lowrank_rows(rng, bases[2], T_q * H, 0.3, q)
        w = _weights(rng, (T_q, H), "domains")
        if with_anchor:
            qa = np.empty((H, d), np.uint16)
            _lowrank_rows(rng, bases[2], H, 0.3, qa)
            out.update(q_anchor=qa, w_anchor=_weights(rng, (H,), "domains"))
    else:
        raise ValueError(f"unknown key recipe {wl.keys!r}")
    hr = wl.head_rank if head_rank is None else head_rank
    if hr > 0:
        # replace the query heads by mixtures of hr latent rows per query row
        lat = np.empty((T_q * hr, d), np.uint16)
        if wl.keys == "gauss":
            _gauss_rows(rng, T_q * hr, d, 1.0 / np.sqrt(128.0), lat)
        else:
            _lowrank_rows(rng, U if wl.keys == "lowrank" else bases[2], T_q * hr, 0.3, lat)
        A = rng.standard_normal((H, hr)) / np.sqrt(hr)
        _mix_heads(rng, lat, A, q)
        if with_anchor:
            la = np.empty((hr, d), np.uint16)
            if wl.keys == "gauss":
                _gauss_rows(rng, hr, d, 1.0 / np.sqrt(128.0), la)
            else:
                _lowrank_rows(rng, U if wl.keys == "lowrank" else bases[2], hr, 0.3, la)
            qa = np.empty((H, d), np.uint16)
            _mix_heads(rng, la, A, qa)
            out["q_anchor"] = qa
    out.update(q=q.reshape(T_q, H, d), w=w, k=k, q_offset=q_offset, T_q=T_q, T_k=T_k,
               H=H, d=d, topk=wl.topk)
    return out


E4M3_MAX = 448.0


def quantize_e4m3_rows(bits: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """FP8 E4M3 codes and one fp32 scale per row of bf16 bit patterns (..., d).

    scale = max|row| / 448 (1 for an all-zero row); codes = E4M3(value / scale)
    rounded to nearest (torch's float8_e4m3fn conversion), so that the row's
    largest magnitude maps to the largest finite code.
    """
    import torch
    vals = bf16_bits_to_f32(bits).astype(np.float32)
    amax = np.abs(vals).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    x = np.clip(vals / scale[..., None], -E4M3_MAX, E4M3_MAX).astype(np.float32)
    codes = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def make_prefill_fp8(wl: Workload | str, **kw) -> dict:
    """make_prefill's inputs stored as FP8: q8 (T_q,H,d) and k8 (T_k,d) E4M3
    codes with per-row fp32 scales q_scale (T_q,H) and k_scale (T_k,); the
    bf16 inputs the codes were made from stay under q / k."""
    x = make_prefill(wl, **kw)
    x["q8"], x["q_scale"] = quantize_e4m3_rows(x["q"])
    x["k8"], x["k_scale"] = quantize_e4m3_rows(x["k"])
    return x


def make_decode(wl: Workload | str, *, B: int | None = None, t_cap: int | None = None,
                seq_len=None, seed: int | None = None) -> dict:
    """Generate B independent decode problems: q (B,H,d), w (B,H), k (B,t_cap,d).

    ``seq_len`` (B,) int32 gives each sequence's cache length (default: all
    t_cap).  Keys past a sequence's length are still drawn so the buffer is
    fully defined.
    """
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    B = wl.B if B is None else B
    t_cap = wl.t_cap if t_cap is None else t_cap
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    H, d = wl.H, wl.d
    k = np.empty((B * t_cap, d), np.uint16)
    q = np.empty((B * H, d), np.uint16)
    if wl.keys == "gauss":
        _gauss_rows(rng, B * t_cap, d, 1.0 / np.sqrt(128.0), k)
        _gauss_rows(rng, B * H, d, 1.0 / np.sqrt(128.0), q)
    else:
        U = _basis(rng, d, wl.rank)
        _lowrank_rows(rng, U, B * t_cap, 0.3, k)
        _lowrank_rows(rng, U, B * H, 0.3, q)
    w = _weights(rng, (B, H), wl.keys)
    if seq_len is None:
        seq_len = np.full(B, t_cap, np.int32)
    seq_len = np.asarray(seq_len, np.int32)
    if seq_len.shape != (B,) or seq_len.min(initial=0) < 0 or seq_len.max(initial=0) > t_cap:
        raise ValueError("seq_len must be (B,) with 0 <= len <= t_cap")
    return dict(q=q.reshape(B, H, d), w=w, k=k.reshape(B, t_cap, d), seq_len=seq_len,
                B=B, t_cap=t_cap, H=H, d=d, topk=wl.topk)


def make_integer_prefill(seed: int, T: int, H: int, d: int, lo: int = -2, hi: int = 2,
                         q_offset: int = 0, T_q: int | None = None) -> dict:
    """Small integer-valued inputs (q, k, w in [lo, hi]); exact in bf16 and fp64."""
    rng = np.random.Generator(np.random.PCG64(seed))
    T_q = T - q_offset if T_q is None else T_q
    q = rng.integers(lo, hi + 1, size=(T_q, H, d)).astype(np.float64)
    k = rng.integers(lo, hi + 1, size=(T, d)).astype(np.float64)
    w = rng.integers(lo, hi + 1, size=(T_q, H)).astype(np.float32)
    return dict(q=bf16_bits_from_f64(q).reshape(T_q, H, d), w=w,
                k=bf16_bits_from_f64(k).reshape(T, d), q_offset=q_offset, T_q=T_q, T_k=T,
                H=H, d=d)


def random_distinct_keys(seed: int, lo: int, hi: int, n: int, exclude=None) -> np.ndarray:
    """``n`` distinct key ids drawn uniformly from [lo, hi), avoiding ``exclude``.

    Returned in draw order as int32.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    taken = set() if exclude is None else {int(x) for x in np.asarray(exclude).ravel()}
    if hi - lo - len([x for x in taken if lo <= x < hi]) < n:
        raise ValueError("not enough keys to draw from")
    out = []
    while len(out) < n:
        cand = rng.integers(lo, hi, size=2 * (n - len(out)) + 16)
        for c in cand.tolist():
            if c not in taken:
                taken.add(c)
                out.append(c)
                if len(out) == n:
                    break
    return np.asarray(out, np.int32)
