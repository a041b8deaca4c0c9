"""The C-ABI library: it loads, exports every symbol the header declares, sizes
workspaces and rejects bad arguments on the host (no GPU needed: validation runs
before anything is enqueued)."""
import ctypes
import os
import re
import subprocess

import pytest

from long_context_token_b200 import build, hs2, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return hs2.lib()


def header_symbols():
    text = open(os.path.join(ROOT, "include", "hs2.h")).read()
    return sorted(set(re.findall(r"HS2_API\s+[\w\s\*]+?\b(hs2_\w+)\s*\(", text)))


def test_library_exports_every_header_symbol(L):
    syms = header_symbols()
    assert len(syms) >= 9 and set(syms) == set(hs2.EXPORTS)
    nm = subprocess.run(["nm", "-D", "--defined-only", hs2.lib_path()], capture_output=True,
                        text=True, check=True).stdout
    exported = set(re.findall(r"\bT (hs2_\w+)", nm))
    assert set(syms) <= exported
    for s in syms:
        assert hasattr(L, s)
    assert L.hs2_abi_version() == 1


def test_status_strings(L):
    for code in range(8):
        assert L.hs2_status_string(code)
    assert L.hs2_status_string(6) == b"sparse index out of range"


@pytest.mark.parametrize("n", sorted(workloads.WORKLOADS))
def test_workspace_sizes_for_every_workload(L, n):
    w = workloads.WORKLOADS[n]
    b = L.hs2_workspace_bytes(w.batch, w.n_q, w.h_q, w.max_len, 128, 1024, int(w.kv == "fp8"))
    # at least the per-key selection buffers, at most a few hundred MB
    assert w.batch * w.n_q * w.max_len * 4 < b < 2 ** 30


@pytest.mark.parametrize("n", sorted(workloads.WORKLOADS))
def test_lse64_offset_lies_inside_the_workspace(L, n):
    """The float64 lse the selection uses: 8-byte aligned, [batch][n_q][h_q] doubles inside
    the workspace, and (size_t)-1 for unsupported sizes."""
    w = workloads.WORKLOADS[n]
    args = (w.batch, w.n_q, w.h_q, w.max_len, 128, 1024, int(w.kv == "fp8"))
    total = L.hs2_workspace_bytes(*args)
    off = L.hs2_workspace_lse64_offset(*args)
    assert off % 8 == 0
    assert off + w.batch * w.n_q * w.h_q * 8 <= total
    assert L.hs2_workspace_lse64_offset(1, 1, 24, 4096, 128, 1024, 0) == 2 ** 64 - 1


@pytest.mark.parametrize("args", [
    (1, 1, 24, 4096, 128, 1024, 0),    # h_q not a multiple of 16
    (1, 1, 144, 4096, 128, 1024, 0),   # h_q > 128
    (1, 65, 16, 4096, 128, 1024, 0),   # n_q > 64
    (1, 1, 16, 4096, 128, 3969, 0),    # window + k_sel > 4096
    (1, 1, 16, 4096, 0, 1024, 0),      # empty window
    (1, 1, 16, 4096, 128, 1024, 2),    # unknown KV type
    (0, 1, 16, 4096, 128, 1024, 0),    # empty batch
    (2048, 64, 16, 4096, 128, 1024, 0),  # 131072 (sequence, token) rows: above the grid's 65535
])
def test_workspace_bytes_rejects_unsupported(L, args):
    assert L.hs2_workspace_bytes(*args) == 0


def _kv(head_dim=128, dtype=0, scales=False, align=0):
    base = 1 << 20
    return hs2.KV(base + align, base + 4096, base if scales else None, base if scales else None,
                  base, 1, 4096, head_dim, dtype)


@pytest.mark.parametrize("kv,q,ws,h,expect", [
    (_kv(), 0, 1 << 20, 16, 1),                  # null q
    (_kv(head_dim=64), 1 << 20, 1 << 20, 16, 2),  # head_dim != 128
    (_kv(), 1 << 20, 1 << 20, 24, 2),            # h_q = 24
    (_kv(), 1 << 20 | 8, 1 << 20, 16, 1),        # misaligned q
    (_kv(align=4), 1 << 20, 1 << 20, 16, 1),     # misaligned k
    (_kv(scales=True), 1 << 20, 1 << 20, 16, 1), # bf16 cache with scales
    (_kv(dtype=1), 1 << 20, 1 << 20, 16, 1),     # fp8 cache without scales
    (_kv(), 1 << 20, 1 << 20, 16, 3),            # workspace too small (size 64)
])
def test_full_attn_select_host_validation(L, kv, q, ws, h, expect):
    code = L.hs2_full_attn_select(q, 1, h, ctypes.byref(kv), 128, 1024, 0.088, 1 << 20,
                                  1 << 20, None, ws, 64, None)
    assert code == expect


def test_sparse_attn_host_validation(L):
    kv = _kv()
    p = 1 << 20
    assert L.hs2_sparse_attn(p, 1, 16, ctypes.byref(kv), p, 0, 0.088, p, p, 1 << 30, None) == 2
    assert L.hs2_sparse_attn(p, 1, 16, ctypes.byref(kv), p, 4097, 0.088, p, p, 1 << 30, None) == 2
    assert L.hs2_sparse_attn(p, 1, 16, ctypes.byref(kv), None, 8, 0.088, p, p, 1 << 30, None) == 1
    assert L.hs2_sparse_attn(p, 1, 16, ctypes.byref(kv), p, 8, 0.088, p, p, 16, None) == 3
    assert L.hs2_check_device_status(None, None) == 1


@pytest.mark.parametrize("kv,kn,nn,lens,ws,wsb,expect", [
    (_kv(), 0, 1, 1 << 20, 1 << 20, 4096, 1),                 # null k_new
    (_kv(), 1 << 20, 1, 0, 1 << 20, 4096, 1),                 # null lens
    (_kv(), 1 << 20, 0, 1 << 20, 1 << 20, 4096, 2),           # n_new = 0
    (_kv(), 1 << 20, 65, 1 << 20, 1 << 20, 4096, 2),          # n_new > 64
    (_kv(), 1 << 20 | 8, 1, 1 << 20, 1 << 20, 4096, 1),       # misaligned k_new
    (_kv(dtype=1), 1 << 20, 1, 1 << 20, 1 << 20, 4096, 1),    # fp8 cache without scales
    (_kv(head_dim=64), 1 << 20, 1, 1 << 20, 1 << 20, 4096, 2),  # head_dim != 128
    (_kv(), 1 << 20, 1, 1 << 20, 1 << 20, 64, 3),             # workspace too small
])
def test_kv_append_rejects_bad_arguments(L, kv, kn, nn, lens, ws, wsb, expect):
    code = L.hs2_kv_append(kn, 1 << 20, nn, ctypes.byref(kv), lens, ws, wsb, None)
    assert code == expect


@pytest.mark.parametrize("block,k_sel,idx,max_len,expect", [
    (1, 1024, 1 << 20, 4096, 2),        # block < 2
    (0, 1024, 1 << 20, 4096, 2),        # block < 2
    (48, 1024, 1 << 20, 4096, 2),       # k_sel not a multiple of block
    (2, 3968, 1 << 20, 4096, 2),        # more than 1024 blocks kept
    (64, 1024, 1 << 20, 1 << 24, 2),    # 262144 block keys do not fit shared memory
    (64, 1024, 0, 4096, 1),             # null idx
])
def test_block_selection_host_validation(L, block, k_sel, idx, max_len, expect):
    base = 1 << 20
    kv = hs2.KV(base, base + 4096, None, None, base, 1, max_len, 128, 0)
    p = 1 << 20
    huge = 1 << 60  # passes the workspace-size check; nothing is dereferenced on the host
    assert L.hs2_full_attn_select_blocks(p, 1, 16, ctypes.byref(kv), 128, k_sel, block, 0.088,
                                         p, idx, None, p, huge, None) == expect
    assert L.hs2_select_blocks(p, 1, 16, ctypes.byref(kv), 128, k_sel, block, 0.088, idx, p,
                               huge, None) == expect


@pytest.mark.parametrize("args", [
    (1, 512, 16, 4096, 1),        # FP8 cache
    (1, 512, 24, 4096, 0),        # h_q not supported
    (1, 0, 16, 4096, 0),          # empty chunk
    (1, 5000, 16, 4096, 0),       # chunk longer than the cache
    (1, 65537, 16, 1 << 20, 0),   # chunk above 65536 tokens
    (0, 512, 16, 4096, 0),        # empty batch
    (1, 65536, 128, 65536, 0),    # 65536 row groups of one token: above the grid's 65535
])
def test_prefill_workspace_rejects_unsupported(L, args):
    assert L.hs2_prefill_workspace_bytes(*args) == 0


def test_prefill_accepts_the_largest_chunk(L):
    # 65536 tokens at 16 heads: 8192 groups of 8 tokens
    assert L.hs2_prefill_workspace_bytes(1, 65536, 16, 65536, 0) > 0


def test_prefill_workspace_holds_the_partials(L):
    # 4096 tokens x h16 in groups of 8: 512 CTAs, one split; partials 4096 * 16 * 130 floats
    n = L.hs2_prefill_workspace_bytes(1, 4096, 16, 131072, 0)
    assert 4096 * 16 * 130 * 4 <= n < 4096 * 16 * 130 * 4 + 4096
    # a short chunk (one CTA of rows) is split along the keys to fill the GPU, up to 32
    # splits: 32 partials per row
    assert L.hs2_prefill_workspace_bytes(1, 8, 16, 131072, 0) >= 8 * 16 * 130 * 4 * 32


def test_prefill_host_validation(L):
    base = 1 << 20
    kv = hs2.KV(base, base + 4096, None, None, base, 1, 4096, 128, 0)
    kv8 = hs2.KV(base, base + 4096, base, base, base, 1, 4096, 128, 1)
    p = 1 << 20
    assert L.hs2_prefill_attn(None, 64, 16, ctypes.byref(kv), 0.088, p, None, p, 1 << 30, None) == 1
    assert L.hs2_prefill_attn(p, 64, 16, ctypes.byref(kv8), 0.088, p, None, p, 1 << 30, None) == 2
    assert L.hs2_prefill_attn(p, 64, 24, ctypes.byref(kv), 0.088, p, None, p, 1 << 30, None) == 2
    assert L.hs2_prefill_attn(p | 8, 64, 16, ctypes.byref(kv), 0.088, p, None, p, 1 << 30, None) == 1
    assert L.hs2_prefill_attn(p, 64, 16, ctypes.byref(kv), 0.088, p, None, p, 64, None) == 3
