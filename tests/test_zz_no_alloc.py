"""hs2_sparse_attn_noalloc, the sparse-layer entry point for callers that cannot
allocate device memory (its scratch is a fixed array inside the library).

It must give the same output as hs2_sparse_attn, which works in a caller-allocated
workspace, on consecutive calls that reuse the shared array, and must refuse sizes
that do not fit in that array.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from long_context_token_b200 import hs2, workloads


@pytest.mark.gpu
@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(kv):
    L = hs2.lib()
    dev = torch.device("cuda:0")
    inp = workloads.make_inputs(2, 5000, n_q=1, h_q=16, kv=kv, n_sparse=2, seed=131,
                                lens=[5000, 3001])
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev),
                      None if inp.k_scale is None else inp.k_scale.to(dev),
                      None if inp.v_scale is None else inp.v_scale.to(dev))
    ws = hs2.alloc_workspace(cache, 1, 16)
    _, idx, _ = hs2.full_attn_select(inp.q.to(dev), cache, workspace=ws)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    tol = 2e-3 if kv == "bf16" else 1e-2
    for layer in range(2):  # two calls in a row share the library's array
        ql = inp.q_layers[layer].to(dev)
        want = hs2.sparse_attn(ql, cache, idx, ws, inp.sm_scale)
        got = torch.full_like(want, float("nan"))
        code = L.hs2_sparse_attn_noalloc(ql.data_ptr(), 1, 16, cache.ref(), idx.data_ptr(),
                                         idx.shape[2], ctypes.c_float(inp.sm_scale),
                                         got.data_ptr(), status.data_ptr(), stream)
        assert code == 0
        torch.cuda.synchronize()
        err = (got - want).abs().max().item()
        assert err <= tol, f"layer {layer}: max-abs difference {err}"
    assert status.item() == 0
    assert hs2.check_device_status(ws) == 0


@pytest.mark.gpu
def test_noalloc_rejects_sizes_beyond_its_array():
    L = hs2.lib()
    dev = torch.device("cuda:0")
    k = torch.zeros(1, 4096, 128, dtype=torch.bfloat16, device=dev)
    lens = torch.full((1,), 4096, dtype=torch.int32, device=dev)
    cache = hs2.Cache(k, k.clone(), lens)
    q = torch.zeros(1, 64, 128, 128, dtype=torch.bfloat16, device=dev)
    idx = torch.zeros(1, 64, 4096, dtype=torch.int32, device=dev)
    out = torch.zeros(1, 64, 128, 128, dtype=torch.float32, device=dev)
    code = L.hs2_sparse_attn_noalloc(q.data_ptr(), 64, 128, cache.ref(), idx.data_ptr(), 4096,
                                     ctypes.c_float(0.088), out.data_ptr(), None,
                                     torch.cuda.current_stream().cuda_stream)
    assert code == 3  # HS2_ERR_WORKSPACE_TOO_SMALL, nothing enqueued
    assert torch.all(out == 0)


def _small_cache(batch, dev, max_len=2048):
    k = torch.randn(batch, max_len, 128, device=dev).to(torch.bfloat16)
    lens = torch.full((batch,), max_len, dtype=torch.int32, device=dev)
    return hs2.Cache(k, k.clone(), lens)


@pytest.mark.gpu
def test_noalloc_size_limit_boundary():
    """B*n_q*h_q = 448 fits the 4 MiB array at 1152 indices; 464 does not."""
    L = hs2.lib()
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream().cuda_stream
    for batch, want in ((28, 0), (29, 3)):  # h_q 16: 448 and 464
        cache = _small_cache(batch, dev)
        q = torch.randn(batch, 1, 16, 128, device=dev).to(torch.bfloat16)
        idx = torch.arange(1152, dtype=torch.int32, device=dev).repeat(batch, 1, 1)
        out = torch.zeros(batch, 1, 16, 128, dtype=torch.float32, device=dev)
        code = L.hs2_sparse_attn_noalloc(q.data_ptr(), 1, 16, cache.ref(), idx.data_ptr(), 1152,
                                         ctypes.c_float(0.088), out.data_ptr(), None, stream)
        torch.cuda.synchronize()
        assert code == want, f"B*n_q*h_q = {batch * 16}: code {code}"
        if want == 0:
            assert torch.isfinite(out).all() and (out != 0).any()
        else:
            assert torch.all(out == 0)  # refused before anything was enqueued


@pytest.mark.gpu
def test_noalloc_reports_index_out_of_range_in_device_status():
    """An index at or past lens[b] is skipped and sets bit 6 (HS2_ERR_INDEX_OUT_OF_RANGE)
    of device_status; with device_status NULL the same call still completes."""
    L = hs2.lib()
    dev = torch.device("cuda:0")
    stream = torch.cuda.current_stream().cuda_stream
    cache = _small_cache(2, dev, max_len=1000)
    cache.lens[1] = 600
    q = torch.randn(2, 1, 16, 128, device=dev).to(torch.bfloat16)
    idx = torch.arange(256, dtype=torch.int32, device=dev).repeat(2, 1, 1)
    idx[1, 0, 7] = 600  # == lens[1]: out of range
    out = torch.zeros(2, 1, 16, 128, dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    code = L.hs2_sparse_attn_noalloc(q.data_ptr(), 1, 16, cache.ref(), idx.data_ptr(), 256,
                                     ctypes.c_float(0.088), out.data_ptr(), status.data_ptr(),
                                     stream)
    torch.cuda.synchronize()
    assert code == 0
    assert status.item() == 1 << 6
    assert torch.isfinite(out).all()
    code = L.hs2_sparse_attn_noalloc(q.data_ptr(), 1, 16, cache.ref(), idx.data_ptr(), 256,
                                     ctypes.c_float(0.088), out.data_ptr(), None, stream)
    torch.cuda.synchronize()
    assert code == 0 and torch.isfinite(out).all()
