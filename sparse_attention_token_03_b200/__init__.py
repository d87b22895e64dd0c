"""B200 (sm_100a) lightning-indexer scoring with exact Top-k.

Python binding of libdsa_index.so (include/dsa_index.h).  This module only
marshals arguments: it checks dtypes, shapes, devices and contiguity of torch
tensors, allocates outputs and the workspace through torch, and passes raw
pointers plus the current CUDA stream to the C ABI.  Every step of the
computation runs in the library's CUDA kernels; there is no fallback.
"""

from __future__ import annotations

import ctypes
from pathlib import Path

import torch

from . import build as _build

__all__ = [
    "DSAError", "lib", "dsa_index_prefill", "dsa_index_prefill_fp8", "dsa_index_decode", "dsa_index_decode_paged",
    "dsa_index_prefill_workspace_bytes", "dsa_index_decode_workspace_bytes",
    "dsa_index_device_status", "dsa_profile_enable", "dsa_profile_read",
    "dsa_index_decode_noalloc", "dsa_index_decode_noalloc_status", "dsa_index_prefill_pruned",
    "dsa_index_prefill_pruned_workspace_bytes", "dsa_index_prefill_pruned_survivors",
    "dsa_index_prefill_host", "dsa_index_prefill_host_workspace_bytes", "dsa_test_inject_wait_timeout",
    "dsa_index_seeds_from_history", "dsa_index_seeds_from_history_workspace_bytes",
    "dsa_index_prefill_paged", "dsa_index_prefill_paged_workspace_bytes",
    "dsa_index_prefill_pruned_paged", "dsa_index_prefill_pruned_paged_workspace_bytes",
]

DSA_OK = 0
STATUS_NAMES = {
    -1: "DSA_EINVAL", -2: "DSA_EUNSUPPORTED", -3: "DSA_EWORKSPACE", -4: "DSA_ESEED",
    -5: "DSA_ECUDA", -6: "DSA_EDEVICE",
}


class DSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def lib(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libdsa_index.so (building it first if it is missing or stale)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if build_if_missing and _build.stale():
            _build.build()
        if not path.exists():
            raise RuntimeError(f"{path} is missing; run sparse_attention_token_03_b200/build.py")
        L = ctypes.CDLL(str(path))
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        L.dsa_last_error_string.restype = ctypes.c_char_p
        L.dsa_index_prefill_workspace_bytes.argtypes = [I64, I64, I, I, I]
        L.dsa_index_prefill_workspace_bytes.restype = SZ
        L.dsa_index_prefill.argtypes = [P, P, P, I64, I64, I64, I, I, I, P, P, P, SZ, P]
        L.dsa_index_prefill.restype = I
        L.dsa_index_prefill_fp8.argtypes = [P, P, P, P, P, I64, I64, I64, I, I, I, P, P, P, SZ, P]
        L.dsa_index_prefill_fp8.restype = I
        L.dsa_index_prefill_host_workspace_bytes.argtypes = [I64, I64, I, I, I]
        L.dsa_index_prefill_host_workspace_bytes.restype = SZ
        L.dsa_index_prefill_host.argtypes = [P, P, P, I64, I64, I64, I, I, I, P, P, P, SZ, P]
        L.dsa_index_prefill_host.restype = I
        L.dsa_index_decode_workspace_bytes.argtypes = [I, I64, I, I, I]
        L.dsa_index_decode_workspace_bytes.restype = SZ
        L.dsa_index_decode.argtypes = [P, P, P, P, I, I64, I, I, I, P, P, P, SZ, P]
        L.dsa_index_decode.restype = I
        L.dsa_index_decode_paged.argtypes = [P, P, P, I64, I, P, I, P, I, I, I, I, P, P, P, SZ, P]
        L.dsa_index_decode_paged.restype = I
        L.dsa_index_prefill_pruned_workspace_bytes.argtypes = [I64, I64, I, I, I, I]
        L.dsa_index_prefill_pruned_workspace_bytes.restype = SZ
        L.dsa_index_prefill_pruned.argtypes = [P, P, P, I64, I64, I64, I, I, I, P, I, P, P, P, P, SZ, P]
        L.dsa_index_prefill_pruned.restype = I
        L.dsa_index_prefill_pruned_survivors.argtypes = [P, I64, I64, I64, I, I, I, I, P, P, P, P]
        L.dsa_index_prefill_pruned_survivors.restype = I
        L.dsa_index_prefill_paged_workspace_bytes.argtypes = [I64, I64, I, I, I]
        L.dsa_index_prefill_paged_workspace_bytes.restype = SZ
        L.dsa_index_prefill_paged.argtypes = [P, P, P, I64, I, P, I64, I64, I64, I, I, I, P, P, P, SZ, P]
        L.dsa_index_prefill_paged.restype = I
        L.dsa_index_prefill_pruned_paged_workspace_bytes.argtypes = [I64, I64, I, I, I, I]
        L.dsa_index_prefill_pruned_paged_workspace_bytes.restype = SZ
        L.dsa_index_prefill_pruned_paged.argtypes = [P, P, P, I64, I, P, I64, I64, I64, I, I, I, P, I, P, P, P, P,
                                                     SZ, P]
        L.dsa_index_prefill_pruned_paged.restype = I
        L.dsa_index_seeds_from_history_workspace_bytes.argtypes = [I64]
        L.dsa_index_seeds_from_history_workspace_bytes.restype = SZ
        L.dsa_index_seeds_from_history.argtypes = [P, I64, I, I64, I, P, P, SZ, P]
        L.dsa_index_seeds_from_history.restype = I
        L.dsa_index_decode_noalloc.argtypes = [P, P, P, P, I, I64, I, I, I, P, P, P]
        L.dsa_index_decode_noalloc.restype = I
        L.dsa_index_decode_noalloc_status.argtypes = [P, P]
        L.dsa_index_decode_noalloc_status.restype = I
        L.dsa_index_device_status.argtypes = [P, P, P]
        L.dsa_index_device_status.restype = I
        L.dsa_test_inject_wait_timeout.argtypes = [I64]
        L.dsa_test_inject_wait_timeout.restype = I
        L.dsa_profile_enable.argtypes = [I]
        L.dsa_profile_enable.restype = I
        L.dsa_profile_read.argtypes = [P, P, I, P]
        L.dsa_profile_read.restype = I
        _lib = L
    return _lib


def _check(rc: int):
    if rc != DSA_OK:
        raise DSAError(rc, lib().dsa_last_error_string().decode())


def _need(t: torch.Tensor, name: str, dtype, ndim: int, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got shape {tuple(t.shape)}")
    if t.device.type != "cuda" or (device is not None and t.device != device):
        raise ValueError(f"{name} must be on {device or 'a CUDA device'}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def dsa_index_prefill_workspace_bytes(T_q: int, T_k: int, H: int, d: int, topk: int) -> int:
    return int(lib().dsa_index_prefill_workspace_bytes(T_q, T_k, H, d, topk))


def dsa_index_decode_workspace_bytes(B: int, t_cap: int, H: int, d: int, topk: int) -> int:
    return int(lib().dsa_index_decode_workspace_bytes(B, t_cap, H, d, topk))


def _workspace(nbytes: int, device, workspace):
    if workspace is None:
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    _need(workspace, "workspace", torch.uint8, 1, device)
    return workspace


def _outputs(rows: int, topk: int, device, out_idx, out_score):
    if out_idx is None:
        out_idx = torch.empty((rows, topk), dtype=torch.int32, device=device)
    if out_score is None:
        out_score = torch.empty((rows, topk), dtype=torch.float32, device=device)
    _need(out_idx, "out_idx", torch.int32, 2, device)
    _need(out_score, "out_score", torch.float32, 2, device)
    if tuple(out_idx.shape) != (rows, topk) or tuple(out_score.shape) != (rows, topk):
        raise ValueError(f"outputs must be ({rows}, {topk})")
    return out_idx, out_score


def dsa_index_prefill(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, q_offset: int, topk: int,
                      out_idx=None, out_score=None, workspace=None):
    """Exact Top-k of the index score for a causal prefill chunk.

    q (T_q, H, d) bf16, w (T_q, H) fp32, k (T_k, d) bf16, all on one CUDA
    device; row t sits at position q_offset + t.  Returns (out_idx, out_score)
    of shape (T_q, topk): int32 key indices and fp32 scores, sorted.
    """
    dev = k.device
    _need(q, "q", torch.bfloat16, 3, dev)
    _need(w, "w", torch.float32, 2, dev)
    _need(k, "k", torch.bfloat16, 2, dev)
    T_q, H, d = q.shape
    T_k = k.shape[0]
    if tuple(w.shape) != (T_q, H) or k.shape[1] != d:
        raise ValueError("shape mismatch between q (T_q,H,d), w (T_q,H) and k (T_k,d)")
    out_idx, out_score = _outputs(T_q, topk, dev, out_idx, out_score)
    nbytes = dsa_index_prefill_workspace_bytes(T_q, T_k, H, d, topk)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_prefill(q.data_ptr(), w.data_ptr(), k.data_ptr(), int(q_offset), T_q,
                                       T_k, H, d, int(topk), out_idx.data_ptr(),
                                       out_score.data_ptr(), ws.data_ptr(), ws.numel(),
                                       _stream_ptr(dev)))
    return out_idx, out_score


def _codes(t: torch.Tensor, name: str, ndim: int, device) -> torch.Tensor:
    """FP8 E4M3 codes given as uint8 or torch.float8_e4m3fn (viewed as uint8)."""
    if isinstance(t, torch.Tensor) and t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    _need(t, name, torch.uint8, ndim, device)
    return t


def dsa_index_prefill_fp8(q: torch.Tensor, q_scale: torch.Tensor, w: torch.Tensor, k: torch.Tensor,
                          k_scale: torch.Tensor, q_offset: int, topk: int, out_idx=None, out_score=None,
                          workspace=None):
    """Exact Top-k of the index score of a causal chunk on FP8 inputs.

    q (T_q, H, d) and k (T_k, d) hold E4M3 codes (uint8 or float8_e4m3fn) with
    fp32 scales q_scale (T_q, H) and k_scale (T_k,); w (T_q, H) fp32.  Returns
    (out_idx, out_score) of shape (T_q, topk), as dsa_index_prefill.
    """
    dev = k.device
    q = _codes(q, "q", 3, dev)
    k = _codes(k, "k", 2, dev)
    _need(q_scale, "q_scale", torch.float32, 2, dev)
    _need(w, "w", torch.float32, 2, dev)
    _need(k_scale, "k_scale", torch.float32, 1, dev)
    T_q, H, d = q.shape
    T_k = k.shape[0]
    if tuple(w.shape) != (T_q, H) or tuple(q_scale.shape) != (T_q, H) or k.shape[1] != d or \
            k_scale.shape[0] != T_k:
        raise ValueError("shape mismatch between q, q_scale, w, k and k_scale")
    out_idx, out_score = _outputs(T_q, topk, dev, out_idx, out_score)
    ws = _workspace(dsa_index_prefill_workspace_bytes(T_q, T_k, H, d, topk), dev, workspace)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_prefill_fp8(q.data_ptr(), q_scale.data_ptr(), w.data_ptr(), k.data_ptr(),
                                           k_scale.data_ptr(), int(q_offset), T_q, T_k, H, d, int(topk),
                                           out_idx.data_ptr(), out_score.data_ptr(), ws.data_ptr(),
                                           ws.numel(), _stream_ptr(dev)))
    return out_idx, out_score


def dsa_index_prefill_host_workspace_bytes(T_q: int, T_k: int, H: int, d: int, topk: int) -> int:
    return int(lib().dsa_index_prefill_host_workspace_bytes(T_q, T_k, H, d, topk))


def _need_host(t: torch.Tensor, name: str, dtype, ndim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype or t.dim() != ndim:
        raise TypeError(f"{name} must be a {ndim}-dim {dtype} tensor, got {t.dtype} {tuple(t.shape)}")
    if t.device.type != "cpu" or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous host (CPU) tensor")


def dsa_index_prefill_host(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, q_offset: int, topk: int,
                           out_idx=None, out_score=None, workspace=None, device=None):
    """dsa_index_prefill from host buffers, with the copies pipelined.

    q (T_q, H, d) bf16, w (T_q, H) fp32, k (T_k, d) bf16 are CPU tensors
    (page-locked ones let the copies overlap the kernels); the outputs are
    CPU tensors (T_q, topk) (page-locked ones are allocated when not given).
    The work is queued on the current stream of ``device`` (default: the
    current CUDA device); the outputs are complete after that stream is
    synchronised.
    """
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _need_host(q, "q", torch.bfloat16, 3)
    _need_host(w, "w", torch.float32, 2)
    _need_host(k, "k", torch.bfloat16, 2)
    T_q, H, d = q.shape
    T_k = k.shape[0]
    if tuple(w.shape) != (T_q, H) or k.shape[1] != d:
        raise ValueError("shape mismatch between q (T_q,H,d), w (T_q,H) and k (T_k,d)")
    if out_idx is None:
        out_idx = torch.empty((T_q, topk), dtype=torch.int32).pin_memory()
    if out_score is None:
        out_score = torch.empty((T_q, topk), dtype=torch.float32).pin_memory()
    _need_host(out_idx, "out_idx", torch.int32, 2)
    _need_host(out_score, "out_score", torch.float32, 2)
    if tuple(out_idx.shape) != (T_q, topk) or tuple(out_score.shape) != (T_q, topk):
        raise ValueError(f"outputs must be ({T_q}, {topk})")
    nbytes = dsa_index_prefill_host_workspace_bytes(T_q, T_k, H, d, topk)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_prefill_host(q.data_ptr(), w.data_ptr(), k.data_ptr(), int(q_offset), T_q,
                                            T_k, H, d, int(topk), out_idx.data_ptr(),
                                            out_score.data_ptr(), ws.data_ptr(), ws.numel(),
                                            _stream_ptr(dev)))
    return out_idx, out_score


class _Stats(ctypes.Structure):
    _fields_ = [("screened_pairs", ctypes.c_int64), ("survivor_pairs", ctypes.c_int64),
                ("refined_pairs", ctypes.c_int64), ("records", ctypes.c_int64),
                ("recovered_rows", ctypes.c_int64), ("bypassed_rows", ctypes.c_int64),
                ("shared_keys", ctypes.c_int64)]


def dsa_index_prefill_pruned_workspace_bytes(T_q: int, T_k: int, H: int, d: int, topk: int,
                                             n_seed: int) -> int:
    return int(lib().dsa_index_prefill_pruned_workspace_bytes(T_q, T_k, H, d, topk, n_seed))


def dsa_index_prefill_pruned(q: torch.Tensor, w: torch.Tensor, k: torch.Tensor, q_offset: int,
                             topk: int, seed_idx: torch.Tensor, out_idx=None, out_score=None,
                             workspace=None, stats: bool = False):
    """Exact Top-k of a causal prefill chunk with DoSA certified pruning.

    Same result as dsa_index_prefill; seed_idx (n_seed,) int32 on the device
    lists distinct keys visible to every row (0 <= seed < q_offset).  With
    stats=True the call synchronises and also returns a dict of counters.
    """
    dev = k.device
    _need(q, "q", torch.bfloat16, 3, dev)
    _need(w, "w", torch.float32, 2, dev)
    _need(k, "k", torch.bfloat16, 2, dev)
    _need(seed_idx, "seed_idx", torch.int32, 1, dev)
    T_q, H, d = q.shape
    T_k = k.shape[0]
    n_seed = seed_idx.shape[0]
    if tuple(w.shape) != (T_q, H) or k.shape[1] != d:
        raise ValueError("shape mismatch between q (T_q,H,d), w (T_q,H) and k (T_k,d)")
    out_idx, out_score = _outputs(T_q, topk, dev, out_idx, out_score)
    nbytes = dsa_index_prefill_pruned_workspace_bytes(T_q, T_k, H, d, topk, max(n_seed, 1))
    ws = _workspace(nbytes, dev, workspace)
    st = _Stats()
    with torch.cuda.device(dev):
        _check(lib().dsa_index_prefill_pruned(q.data_ptr(), w.data_ptr(), k.data_ptr(), int(q_offset),
                                              T_q, T_k, H, d, int(topk), seed_idx.data_ptr(), n_seed,
                                              out_idx.data_ptr(), out_score.data_ptr(),
                                              ctypes.byref(st) if stats else None, ws.data_ptr(),
                                              ws.numel(), _stream_ptr(dev)))
    if stats:
        return out_idx, out_score, {f: int(getattr(st, f)) for f, _ in _Stats._fields_}
    return out_idx, out_score


def dsa_index_prefill_paged_workspace_bytes(T_q: int, T_k: int, H: int, d: int, topk: int) -> int:
    return int(lib().dsa_index_prefill_paged_workspace_bytes(T_q, T_k, H, d, topk))


def dsa_index_prefill_pruned_paged_workspace_bytes(T_q: int, T_k: int, H: int, d: int, topk: int,
                                                   n_seed: int) -> int:
    return int(lib().dsa_index_prefill_pruned_paged_workspace_bytes(T_q, T_k, H, d, topk, n_seed))


def _paged_args(q, w, k_pages, block_table, dev):
    _need(q, "q", torch.bfloat16, 3, dev)
    _need(w, "w", torch.float32, 2, dev)
    _need(k_pages, "k_pages", torch.bfloat16, 3, dev)
    _need(block_table, "block_table", torch.int32, 1, dev)
    T_q, H, d = q.shape
    n_pages, page_size, dk = k_pages.shape
    if tuple(w.shape) != (T_q, H) or dk != d:
        raise ValueError("shape mismatch between q (T_q,H,d), w (T_q,H) and k_pages (n_pages,page_size,d)")
    return T_q, H, d, n_pages, page_size


def dsa_index_prefill_paged(q: torch.Tensor, w: torch.Tensor, k_pages: torch.Tensor, block_table: torch.Tensor,
                            q_offset: int, topk: int, T_k: int | None = None, out_idx=None, out_score=None,
                            workspace=None):
    """dsa_index_prefill over a paged key cache: key s of the sequence is
    k_pages[block_table[s // page_size], s % page_size].  T_k defaults to
    q_offset + T_q."""
    dev = k_pages.device
    T_q, H, d, n_pages, page_size = _paged_args(q, w, k_pages, block_table, dev)
    T_k = int(q_offset) + T_q if T_k is None else int(T_k)
    if block_table.shape[0] * page_size < T_k:
        raise ValueError("block_table does not cover T_k keys")
    out_idx, out_score = _outputs(T_q, topk, dev, out_idx, out_score)
    ws = _workspace(dsa_index_prefill_paged_workspace_bytes(T_q, T_k, H, d, topk), dev, workspace)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_prefill_paged(q.data_ptr(), w.data_ptr(), k_pages.data_ptr(), n_pages, page_size,
                                             block_table.data_ptr(), int(q_offset), T_q, T_k, H, d, int(topk),
                                             out_idx.data_ptr(), out_score.data_ptr(), ws.data_ptr(), ws.numel(),
                                             _stream_ptr(dev)))
    return out_idx, out_score


def dsa_index_prefill_pruned_paged(q: torch.Tensor, w: torch.Tensor, k_pages: torch.Tensor,
                                   block_table: torch.Tensor, q_offset: int, topk: int, seed_idx: torch.Tensor,
                                   T_k: int | None = None, out_idx=None, out_score=None, workspace=None,
                                   stats: bool = False):
    """dsa_index_prefill_pruned over a paged key cache (see
    dsa_index_prefill_paged for the page layout)."""
    dev = k_pages.device
    T_q, H, d, n_pages, page_size = _paged_args(q, w, k_pages, block_table, dev)
    _need(seed_idx, "seed_idx", torch.int32, 1, dev)
    T_k = int(q_offset) + T_q if T_k is None else int(T_k)
    if block_table.shape[0] * page_size < T_k:
        raise ValueError("block_table does not cover T_k keys")
    n_seed = seed_idx.shape[0]
    out_idx, out_score = _outputs(T_q, topk, dev, out_idx, out_score)
    ws = _workspace(dsa_index_prefill_pruned_paged_workspace_bytes(T_q, T_k, H, d, topk, max(n_seed, 1)), dev,
                    workspace)
    st = _Stats()
    with torch.cuda.device(dev):
        _check(lib().dsa_index_prefill_pruned_paged(q.data_ptr(), w.data_ptr(), k_pages.data_ptr(), n_pages,
                                                    page_size, block_table.data_ptr(), int(q_offset), T_q, T_k,
                                                    H, d, int(topk), seed_idx.data_ptr(), n_seed,
                                                    out_idx.data_ptr(), out_score.data_ptr(),
                                                    ctypes.byref(st) if stats else None, ws.data_ptr(),
                                                    ws.numel(), _stream_ptr(dev)))
    if stats:
        return out_idx, out_score, {f: int(getattr(st, f)) for f, _ in _Stats._fields_}
    return out_idx, out_score


def dsa_index_prefill_pruned_survivors(workspace: torch.Tensor, T_q: int, T_k: int, q_offset: int, H: int,
                                       d: int, topk: int, n_seed: int):
    """The screen's decisions of the last pruned call on `workspace` (same sizes).

    Returns (mask (T_q, ceil(T_k/32)) int32 bit words, tau (T_q,) fp32,
    row_state (T_q,) int32) on the workspace's device.
    """
    dev = workspace.device
    _need(workspace, "workspace", torch.uint8, 1, dev)
    mask = torch.empty((T_q, (T_k + 31) // 32), dtype=torch.int32, device=dev)
    tau = torch.empty(T_q, dtype=torch.float32, device=dev)
    state = torch.empty(T_q, dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_prefill_pruned_survivors(workspace.data_ptr(), T_q, T_k, int(q_offset), H, d,
                                                        int(topk), int(n_seed), mask.data_ptr(),
                                                        tau.data_ptr(), state.data_ptr(), _stream_ptr(dev)))
    return mask, tau, state


def dsa_index_seeds_from_history_workspace_bytes(n_keys: int) -> int:
    return int(lib().dsa_index_seeds_from_history_workspace_bytes(int(n_keys)))


def dsa_index_seeds_from_history(prev_idx: torch.Tensor, n_keys: int, n_seed: int, out=None, workspace=None):
    """The n_seed keys below n_keys most often selected in prev_idx.

    prev_idx (n_rows, topk) int32 on the GPU (earlier rows' out_idx, -1
    padding ignored).  Returns (n_seed,) int32 in ascending key order: the
    largest counts, ties to the smaller key.
    """
    dev = prev_idx.device
    _need(prev_idx, "prev_idx", torch.int32, 2, dev)
    n_rows, topk = prev_idx.shape
    if out is None:
        out = torch.empty(n_seed, dtype=torch.int32, device=dev)
    _need(out, "out", torch.int32, 1, dev)
    if out.shape[0] != n_seed:
        raise ValueError(f"out must be ({n_seed},)")
    nbytes = dsa_index_seeds_from_history_workspace_bytes(n_keys)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_seeds_from_history(prev_idx.data_ptr() if n_rows else None, n_rows, max(topk, 1),
                                                  int(n_keys), int(n_seed), out.data_ptr(), ws.data_ptr(),
                                                  ws.numel(), _stream_ptr(dev)))
    return out


def dsa_index_decode(q: torch.Tensor, w: torch.Tensor, k_cache: torch.Tensor,
                     seq_len: torch.Tensor, topk: int, out_idx=None, out_score=None,
                     workspace=None):
    """Exact Top-k for one new query per sequence against its own key cache.

    q (B, H, d) bf16, w (B, H) fp32, k_cache (B, t_cap, d) bf16, seq_len (B,)
    int32 on the same device.  Returns (out_idx, out_score) of shape (B, topk).
    """
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, 3, dev)
    _need(w, "w", torch.float32, 2, dev)
    _need(k_cache, "k_cache", torch.bfloat16, 3, dev)
    _need(seq_len, "seq_len", torch.int32, 1, dev)
    B, H, d = q.shape
    t_cap = k_cache.shape[1]
    if tuple(w.shape) != (B, H) or k_cache.shape[0] != B or k_cache.shape[2] != d or seq_len.shape[0] != B:
        raise ValueError("shape mismatch between q, w, k_cache and seq_len")
    out_idx, out_score = _outputs(B, topk, dev, out_idx, out_score)
    nbytes = dsa_index_decode_workspace_bytes(B, t_cap, H, d, topk)
    ws = _workspace(nbytes, dev, workspace)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_decode(q.data_ptr(), w.data_ptr(), k_cache.data_ptr(),
                                      seq_len.data_ptr(), B, t_cap, H, d, int(topk),
                                      out_idx.data_ptr(), out_score.data_ptr(), ws.data_ptr(),
                                      ws.numel(), _stream_ptr(dev)))
    return out_idx, out_score


def dsa_index_decode_paged(q: torch.Tensor, w: torch.Tensor, k_pages: torch.Tensor,
                           block_table: torch.Tensor, seq_len: torch.Tensor, topk: int, out_idx=None,
                           out_score=None, workspace=None):
    """Exact Top-k for one new query per sequence against a paged key cache.

    q (B, H, d) bf16, w (B, H) fp32, k_pages (n_pages, page_size, d) bf16 (the
    page pool; page_size a multiple of 64), block_table (B, max_blocks) int32
    page ids, seq_len (B,) int32.  Returns (out_idx, out_score) of shape
    (B, topk) with key positions within each sequence.
    """
    dev = k_pages.device
    _need(q, "q", torch.bfloat16, 3, dev)
    _need(w, "w", torch.float32, 2, dev)
    _need(k_pages, "k_pages", torch.bfloat16, 3, dev)
    _need(block_table, "block_table", torch.int32, 2, dev)
    _need(seq_len, "seq_len", torch.int32, 1, dev)
    B, H, d = q.shape
    n_pages, page_size = k_pages.shape[0], k_pages.shape[1]
    max_blocks = block_table.shape[1]
    if tuple(w.shape) != (B, H) or k_pages.shape[2] != d or block_table.shape[0] != B or seq_len.shape[0] != B:
        raise ValueError("shape mismatch between q, w, k_pages, block_table and seq_len")
    out_idx, out_score = _outputs(B, topk, dev, out_idx, out_score)
    ws = _workspace(dsa_index_decode_workspace_bytes(B, max_blocks * page_size, H, d, topk), dev, workspace)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_decode_paged(q.data_ptr(), w.data_ptr(), k_pages.data_ptr(), n_pages, page_size,
                                            block_table.data_ptr(), max_blocks, seq_len.data_ptr(), B, H, d,
                                            int(topk), out_idx.data_ptr(), out_score.data_ptr(), ws.data_ptr(),
                                            ws.numel(), _stream_ptr(dev)))
    return out_idx, out_score


def dsa_index_decode_noalloc(q: torch.Tensor, w: torch.Tensor, k_cache: torch.Tensor,
                             seq_len: torch.Tensor, topk: int, out_idx=None, out_score=None):
    """dsa_index_decode without a workspace: the library's static device
    scratch serves at most 64 sequences, and calls must not overlap on the GPU.
    Pass preallocated outputs to keep the call free of any allocation."""
    dev = k_cache.device
    _need(q, "q", torch.bfloat16, 3, dev)
    _need(w, "w", torch.float32, 2, dev)
    _need(k_cache, "k_cache", torch.bfloat16, 3, dev)
    _need(seq_len, "seq_len", torch.int32, 1, dev)
    B, H, d = q.shape
    t_cap = k_cache.shape[1]
    if tuple(w.shape) != (B, H) or k_cache.shape[0] != B or k_cache.shape[2] != d or seq_len.shape[0] != B:
        raise ValueError("shape mismatch between q, w, k_cache and seq_len")
    out_idx, out_score = _outputs(B, topk, dev, out_idx, out_score)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_decode_noalloc(q.data_ptr(), w.data_ptr(), k_cache.data_ptr(),
                                              seq_len.data_ptr(), B, t_cap, H, d, int(topk),
                                              out_idx.data_ptr(), out_score.data_ptr(),
                                              _stream_ptr(dev)))
    return out_idx, out_score


def dsa_index_decode_noalloc_status(device=None) -> int:
    """Device status word of the last dsa_index_decode_noalloc call on
    ``device`` (default: the current CUDA device); synchronises its current
    stream and allocates nothing."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        _check(lib().dsa_index_decode_noalloc_status(ctypes.byref(st), _stream_ptr(dev)))
    return int(st.value)


def dsa_test_inject_wait_timeout(limit_ns: int) -> None:
    """Arm a one-shot injected wait timeout for the calling thread's next
    scoring launch (tests of the bounded-wait failure path)."""
    _check(lib().dsa_test_inject_wait_timeout(int(limit_ns)))


def dsa_profile_enable(on: bool = True) -> None:
    """Record per-kernel CUDA events inside the library's entry points."""
    _check(lib().dsa_profile_enable(1 if on else 0))


def dsa_profile_read() -> list[tuple[str, float]]:
    """(kernel name, device ms) for each kernel of the calling thread's last call."""
    ms = (ctypes.c_float * 32)()
    names = (ctypes.c_char_p * 32)()
    n = ctypes.c_int(0)
    _check(lib().dsa_profile_read(ms, names, 32, ctypes.byref(n)))
    return [(names[i].decode(), float(ms[i])) for i in range(min(n.value, 32))]


def dsa_index_device_status(workspace: torch.Tensor) -> int:
    """Device status word of the last call that used `workspace` (synchronises)."""
    st = ctypes.c_uint32(0)
    with torch.cuda.device(workspace.device):
        _check(lib().dsa_index_device_status(workspace.data_ptr(), ctypes.byref(st),
                                             _stream_ptr(workspace.device)))
    return int(st.value)
