"""The C ABI library loads and exports every entry point the headers declare;
host-side argument validation answers without touching a GPU."""

import ctypes
import re
from pathlib import Path

import pytest

import sparse_attention_token_03_b200 as dsa

ROOT = Path(__file__).resolve().parent.parent


def declared_symbols():
    names = []
    for h in sorted((ROOT / "include").glob("*.h")):
        text = h.read_text()
        names += re.findall(r"DSA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)
    return names


def test_headers_declare_the_entry_points():
    names = set(declared_symbols())
    for n in ("dsa_index_prefill", "dsa_index_decode", "dsa_index_prefill_workspace_bytes",
              "dsa_index_decode_workspace_bytes", "dsa_last_error_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    L = dsa.lib()
    missing = [n for n in declared_symbols() if not hasattr(L, n)]
    assert not missing, missing


def test_host_validation_without_gpu():
    L = dsa.lib()
    P = ctypes.c_void_p
    dummy = P(16)
    # unsupported head count / width / topk
    assert L.dsa_index_prefill(dummy, dummy, dummy, 0, 4, 4, 48, 128, 8, dummy, dummy, dummy, 1 << 20, None) == -2
    assert L.dsa_index_prefill(dummy, dummy, dummy, 0, 4, 4, 64, 64, 8, dummy, dummy, dummy, 1 << 20, None) == -2
    assert L.dsa_index_prefill(dummy, dummy, dummy, 0, 4, 4, 64, 128, 0, dummy, dummy, dummy, 1 << 20, None) == -2
    assert L.dsa_index_prefill(dummy, dummy, dummy, 0, 4, 4, 64, 128, 4096, dummy, dummy, dummy, 1 << 20, None) == -2
    assert b"topk" in L.dsa_last_error_string()
    # inconsistent sizes
    assert L.dsa_index_prefill(dummy, dummy, dummy, 2, 4, 4, 64, 128, 8, dummy, dummy, dummy, 1 << 20, None) == -1
    assert L.dsa_index_prefill(dummy, dummy, dummy, -1, 4, 8, 64, 128, 8, dummy, dummy, dummy, 1 << 20, None) == -1
    # empty chunk is a no-op
    assert L.dsa_index_prefill(None, None, dummy, 0, 0, 4, 64, 128, 8, None, None, None, 0, None) == 0
    # null pointers
    assert L.dsa_index_prefill(None, dummy, dummy, 0, 4, 4, 64, 128, 8, dummy, dummy, dummy, 1 << 20, None) == -1
    # decode: bad batch
    assert L.dsa_index_decode(dummy, dummy, dummy, dummy, 0, 16, 64, 128, 8, dummy, dummy, dummy, 1 << 20, None) == -1
    assert L.dsa_index_decode(dummy, dummy, dummy, dummy, 4, 16, 64, 100, 8, dummy, dummy, dummy, 1 << 20, None) == -2
    # workspace queries reject unsupported shapes with 0
    assert L.dsa_index_prefill_workspace_bytes(4, 4, 48, 128, 8) == 0
    assert L.dsa_index_decode_workspace_bytes(0, 16, 64, 128, 8) == 0


def test_host_buffer_prefill_validation_without_gpu():
    L = dsa.lib()
    P = ctypes.c_void_p
    dummy = P(256)
    # unsupported heads, inconsistent sizes and null pointers fail before any CUDA call
    assert L.dsa_index_prefill_host(dummy, dummy, dummy, 0, 4, 4, 48, 128, 8, dummy, dummy, dummy, 1 << 30, None) == -2
    assert L.dsa_index_prefill_host(dummy, dummy, dummy, 3, 4, 4, 64, 128, 8, dummy, dummy, dummy, 1 << 30, None) == -1
    assert L.dsa_index_prefill_host(None, dummy, dummy, 0, 4, 4, 64, 128, 8, dummy, dummy, dummy, 1 << 30, None) == -1
    # a workspace below the size query is refused
    need = L.dsa_index_prefill_host_workspace_bytes(4, 4, 64, 128, 8)
    assert need > 0
    assert L.dsa_index_prefill_host(dummy, dummy, dummy, 0, 4, 4, 64, 128, 8, dummy, dummy, dummy, need - 1, None) == -3
    assert b"workspace" in L.dsa_last_error_string()
    # an empty chunk is a no-op; unsupported shapes size to 0
    assert L.dsa_index_prefill_host(None, None, dummy, 0, 0, 4, 64, 128, 8, None, None, None, 0, None) == 0
    assert L.dsa_index_prefill_host_workspace_bytes(4, 4, 64, 128, 4096) == 0


def test_host_buffer_binding_checks_dtypes_without_gpu():
    import torch
    q = torch.zeros((4, 64, 128), dtype=torch.float32)
    w = torch.zeros((4, 64), dtype=torch.float32)
    k = torch.zeros((4, 128), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        dsa.dsa_index_prefill_host(q, w, k, 0, 8, device="cpu")


def test_binding_has_the_header_names():
    # the Python layer is a thin binding with the C ABI's names; the error
    # string is surfaced through DSAError instead of its own function
    hdr = (ROOT / "include" / "dsa_index.h").read_text()
    names = set(re.findall(r"^DSA_API\s+[\w\s\*]+?\b(dsa_\w+)\s*\(", hdr, flags=re.M))
    assert "dsa_index_prefill_host" in names and len(names) >= 12
    missing = sorted(n for n in names - {"dsa_last_error_string"} if not callable(getattr(dsa, n, None)))
    assert not missing, missing
    assert set(dsa.__all__) >= names - {"dsa_last_error_string"}


def test_history_seeds_validation_without_gpu():
    L = dsa.lib()
    P = ctypes.c_void_p
    dummy = P(256)
    need = L.dsa_index_seeds_from_history_workspace_bytes(100_003)
    # counts and a 65536-bin histogram at least; tile prefixes for 98 tiles
    assert need >= 4 * 100_003 + 4 * 65536 and need % 256 == 0
    assert L.dsa_index_seeds_from_history_workspace_bytes(0) == 0
    # n_seed outside [1, n_keys], bad sizes, nulls, short or misaligned workspace
    assert L.dsa_index_seeds_from_history(dummy, 4, 8, 10, 11, dummy, dummy, need, None) == -1
    assert L.dsa_index_seeds_from_history(dummy, 4, 8, 10, 0, dummy, dummy, need, None) == -1
    assert L.dsa_index_seeds_from_history(dummy, -1, 8, 10, 5, dummy, dummy, need, None) == -1
    assert L.dsa_index_seeds_from_history(None, 4, 8, 10, 5, dummy, dummy, need, None) == -1
    assert L.dsa_index_seeds_from_history(dummy, 1 << 30, 8, 10, 5, dummy, dummy, need, None) == -1
    assert L.dsa_index_seeds_from_history(dummy, 4, 8, 10, 5, dummy, P(264), need, None) == -1
    small = L.dsa_index_seeds_from_history_workspace_bytes(10)
    assert L.dsa_index_seeds_from_history(dummy, 4, 8, 10, 5, dummy, dummy, small - 1, None) == -3


def test_paged_prefill_validation_without_gpu():
    L = dsa.lib()
    P = ctypes.c_void_p
    d = P(256)
    need = L.dsa_index_prefill_paged_workspace_bytes(256, 1024, 64, 128, 64)
    # the contiguous call's workspace plus the status block and 1024 gathered keys
    assert need >= L.dsa_index_prefill_workspace_bytes(256, 1024, 64, 128, 64) + 256 + 1024 * 256
    assert L.dsa_index_prefill_pruned_paged_workspace_bytes(256, 1024, 64, 128, 64, 128) >= \
        L.dsa_index_prefill_pruned_workspace_bytes(256, 1024, 64, 128, 64, 128) + 1024 * 256
    # unsupported heads, bad page sizes, null pools and misaligned workspaces fail before any CUDA call
    assert L.dsa_index_prefill_paged(d, d, d, 8, 128, d, 768, 256, 1024, 48, 128, 64, d, d, d, need, None) == -2
    assert L.dsa_index_prefill_paged(d, d, d, 8, 0, d, 768, 256, 1024, 64, 128, 64, d, d, d, need, None) == -1
    assert L.dsa_index_prefill_paged(d, d, None, 8, 128, d, 768, 256, 1024, 64, 128, 64, d, d, d, need, None) == -1
    assert L.dsa_index_prefill_paged(d, d, d, 8, 128, d, 768, 256, 1024, 64, 128, 64, d, d, P(264), need,
                                     None) == -1
    assert L.dsa_index_prefill_paged(d, d, d, 8, 128, d, 768, 256, 1024, 64, 128, 64, d, d, d, 1000, None) == -3
