"""ctypes binding of libhs2 (argument marshalling only; every step runs in the CUDA
library).  PyTorch provides device memory and the current stream.

    cache = Cache(k, v, lens)                        # FP8: Cache(k, v, lens, k_scale, v_scale)
    ws = alloc_workspace(cache, n_q, h_q)
    kv_append(k_new, v_new, cache, ws)               # the new tokens' K/V rows; lens grows
    out, idx, lse = full_attn_select(q, cache, workspace=ws)    # full layer + selection
    out_l = sparse_attn(q_layer, cache, idx, ws)     # one reusing sparse layer
    # comparators and neighbours of the step:
    out, idx, lse = full_attn_select_blocks(q, cache, block=64, workspace=ws)
    out, lse = prefill_attn(q_chunk, cache)          # full layer over a chunk of new tokens

The library is loaded from ``long_context_token_b200/_lib/libhs2.so``.  There is no
fallback: if the library is missing or no CUDA device is present, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libhs2.so")

HS2_KV_BF16 = 0
HS2_KV_FP8_E4M3 = 1

STATUS = {
    0: "HS2_OK", 1: "HS2_ERR_INVALID_ARGUMENT", 2: "HS2_ERR_UNSUPPORTED",
    3: "HS2_ERR_WORKSPACE_TOO_SMALL", 4: "HS2_ERR_CUDA", 5: "HS2_ERR_DEVICE_TIMEOUT",
    6: "HS2_ERR_INDEX_OUT_OF_RANGE", 7: "HS2_ERR_BAD_LENGTH",
}

EXPORTS = ("hs2_workspace_bytes", "hs2_full_attn_select", "hs2_full_attn", "hs2_select",
           "hs2_sparse_attn", "hs2_check_device_status", "hs2_status_string",
           "hs2_last_cuda_error", "hs2_abi_version", "hs2_sparse_attn_noalloc", "hs2_kv_append",
           "hs2_full_attn_select_blocks", "hs2_select_blocks", "hs2_prefill_workspace_bytes",
           "hs2_prefill_attn", "hs2_select_fused", "hs2_workspace_lse64_offset",
           "hs2_debug_stall_waits", "hs2_set_deterministic")


class Hs2Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        self.name = STATUS.get(code, str(code))
        detail = lib().hs2_status_string(code).decode()
        cuda = lib().hs2_last_cuda_error().decode() if code == 4 else ""
        super().__init__(f"{what}: {self.name} ({detail}){' - ' + cuda if cuda else ''}")


class KV(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("lens", ctypes.c_void_p), ("batch", ctypes.c_int32),
                ("max_len", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def lib():
    """Load libhs2 (once).  Raises if the shared library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"libhs2 is not built ({_LIB_PATH} missing); run "
                           "`python -m long_context_token_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    kvp = ctypes.POINTER(KV)
    L.hs2_workspace_bytes.argtypes = [i32] * 7
    L.hs2_workspace_bytes.restype = sz
    L.hs2_full_attn_select.argtypes = [vp, i32, i32, kvp, i32, i32, f32, vp, vp, vp, vp, sz, vp]
    L.hs2_full_attn_select.restype = i32
    L.hs2_full_attn.argtypes = [vp, i32, i32, kvp, i32, i32, f32, vp, vp, vp, sz, vp]
    L.hs2_full_attn.restype = i32
    L.hs2_select.argtypes = [vp, i32, i32, kvp, i32, i32, f32, vp, vp, sz, vp]
    L.hs2_select.restype = i32
    L.hs2_sparse_attn.argtypes = [vp, i32, i32, kvp, vp, i32, f32, vp, vp, sz, vp]
    L.hs2_sparse_attn.restype = i32
    L.hs2_sparse_attn_noalloc.argtypes = [vp, i32, i32, kvp, vp, i32, f32, vp, vp, vp]
    L.hs2_sparse_attn_noalloc.restype = i32
    L.hs2_full_attn_select_blocks.argtypes = [vp, i32, i32, kvp, i32, i32, i32, f32, vp, vp, vp,
                                              vp, sz, vp]
    L.hs2_full_attn_select_blocks.restype = i32
    L.hs2_select_blocks.argtypes = [vp, i32, i32, kvp, i32, i32, i32, f32, vp, vp, sz, vp]
    L.hs2_select_blocks.restype = i32
    L.hs2_prefill_workspace_bytes.argtypes = [i32] * 5
    L.hs2_prefill_workspace_bytes.restype = sz
    L.hs2_prefill_attn.argtypes = [vp, i32, i32, kvp, f32, vp, vp, vp, sz, vp]
    L.hs2_prefill_attn.restype = i32
    L.hs2_kv_append.argtypes = [vp, vp, i32, kvp, vp, vp, sz, vp]
    L.hs2_kv_append.restype = i32
    L.hs2_check_device_status.argtypes = [vp, vp]
    L.hs2_check_device_status.restype = i32
    L.hs2_status_string.argtypes = [i32]
    L.hs2_status_string.restype = ctypes.c_char_p
    L.hs2_last_cuda_error.argtypes = []
    L.hs2_last_cuda_error.restype = ctypes.c_char_p
    L.hs2_abi_version.argtypes = []
    L.hs2_abi_version.restype = i32
    L.hs2_select_fused.argtypes = [i32, i32, i32]
    L.hs2_select_fused.restype = i32
    L.hs2_workspace_lse64_offset.argtypes = [i32] * 7
    L.hs2_workspace_lse64_offset.restype = sz
    L.hs2_debug_stall_waits.argtypes = [i32]
    L.hs2_debug_stall_waits.restype = None
    L.hs2_set_deterministic.argtypes = [i32]
    L.hs2_set_deterministic.restype = None
    _lib = L
    return L


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _check(code: int, what: str):
    if code != 0:
        raise Hs2Error(code, what)


class Cache:
    """The shared KV cache of one hybrid block, resident on the device.

    k, v: [B, max_len, 128] bf16, or uint8 / float8_e4m3fn E4M3 codes with
    k_scale / v_scale float32 [B, max_len]; lens int32 [B]."""

    def __init__(self, k, v, lens, k_scale=None, v_scale=None):
        if k.dtype == torch.float8_e4m3fn:
            k, v = k.view(torch.uint8), v.view(torch.uint8)
        fp8 = k.dtype == torch.uint8
        for name, t in (("k", k), ("v", v), ("lens", lens)):
            if not t.is_cuda or not t.is_contiguous():
                raise ValueError(f"{name} must be a contiguous CUDA tensor")
        if k.shape != v.shape or k.dim() != 3 or k.shape[2] != 128:
            raise ValueError("k and v must be [B, max_len, 128]")
        if not fp8 and k.dtype != torch.bfloat16:
            raise ValueError("k/v must be bfloat16 or E4M3 codes")
        if lens.dtype != torch.int32 or lens.shape != (k.shape[0],):
            raise ValueError("lens must be int32 [B]")
        if fp8:
            for name, t in (("k_scale", k_scale), ("v_scale", v_scale)):
                if t is None or t.dtype != torch.float32 or not t.is_cuda or \
                        t.shape != k.shape[:2] or not t.is_contiguous():
                    raise ValueError(f"{name} must be float32 [B, max_len] on the device")
        elif k_scale is not None or v_scale is not None:
            raise ValueError("bf16 caches take no scales")
        self.k, self.v, self.lens, self.k_scale, self.v_scale = k, v, lens, k_scale, v_scale
        self.dtype = HS2_KV_FP8_E4M3 if fp8 else HS2_KV_BF16
        self._struct = KV(k.data_ptr(), v.data_ptr(), _ptr(k_scale), _ptr(v_scale),
                          lens.data_ptr(), k.shape[0], k.shape[1], 128, self.dtype)

    @property
    def batch(self) -> int:
        return self.k.shape[0]

    @property
    def max_len(self) -> int:
        return self.k.shape[1]

    def ref(self):
        return ctypes.byref(self._struct)


def workspace_bytes(batch: int, n_q: int, h_q: int, max_len: int, window: int = 128,
                    k_sel: int = 1024, fp8: bool = False) -> int:
    n = lib().hs2_workspace_bytes(batch, n_q, h_q, max_len, window, k_sel,
                                  HS2_KV_FP8_E4M3 if fp8 else HS2_KV_BF16)
    if n == 0:
        raise Hs2Error(2, "hs2_workspace_bytes")
    return n


def alloc_workspace(cache: Cache, n_q: int, h_q: int, window: int = 128, k_sel: int = 1024,
                    device=None) -> torch.Tensor:
    """A zero-filled workspace (uint8 tensor) for these sizes."""
    n = workspace_bytes(cache.batch, n_q, h_q, cache.max_len, window, k_sel,
                        cache.dtype == HS2_KV_FP8_E4M3)
    return torch.zeros(n, dtype=torch.uint8, device=device or cache.k.device)


def _check_q(q: torch.Tensor, cache: Cache) -> Tuple[int, int]:
    if q.dtype != torch.bfloat16 or not q.is_cuda or not q.is_contiguous() or q.dim() != 4 \
            or q.shape[0] != cache.batch or q.shape[3] != 128:
        raise ValueError("queries must be contiguous bf16 [B, n_q, h_q, 128] on the device")
    return q.shape[1], q.shape[2]


def default_scale() -> float:
    return float(torch.tensor(1.0 / math.sqrt(128.0), dtype=torch.float32))


def select_fused(cache: "Cache", n_q: int, h_q: int) -> bool:
    """True if full_attn_select runs as one kernel for these sizes (hs2_select_fused)."""
    return bool(lib().hs2_select_fused(n_q, h_q, cache.dtype))


def set_deterministic(on: bool) -> None:
    """Static key chunks in the full layer: bitwise-reproducible runs (hs2_set_deterministic)."""
    lib().hs2_set_deterministic(1 if on else 0)


def workspace_lse64(workspace: torch.Tensor, cache: "Cache", n_q: int, h_q: int,
                    window: int = 128, k_sel: int = 1024) -> torch.Tensor:
    """The float64 lse [batch, n_q, h_q] that the last full layer left in `workspace`
    (a view, not a copy; hs2_workspace_lse64_offset)."""
    off = lib().hs2_workspace_lse64_offset(cache.batch, n_q, h_q, cache.max_len, window,
                                           k_sel, cache.dtype)
    if off == (1 << 64) - 1:
        raise Hs2Error(2, "hs2_workspace_lse64_offset")
    n = cache.batch * n_q * h_q * 8
    return workspace[off:off + n].view(torch.float64).view(cache.batch, n_q, h_q)


def full_attn_select(q: torch.Tensor, cache: Cache, window: int = 128, k_sel: int = 1024,
                     sm_scale: Optional[float] = None, workspace: Optional[torch.Tensor] = None,
                     out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                     lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """Full-attention layer + token selection.  Returns (out, idx, lse)."""
    n_q, h = _check_q(q, cache)
    B = cache.batch
    sm_scale = default_scale() if sm_scale is None else sm_scale
    if workspace is None:
        workspace = alloc_workspace(cache, n_q, h, window, k_sel)
    if out is None:
        out = torch.empty(B, n_q, h, 128, dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty(B, n_q, window + k_sel, dtype=torch.int32, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, n_q, h, dtype=torch.float32, device=q.device)
    code = lib().hs2_full_attn_select(q.data_ptr(), n_q, h, cache.ref(), window, k_sel,
                                      sm_scale, out.data_ptr(), idx.data_ptr(), _ptr(lse),
                                      workspace.data_ptr(), workspace.numel(), _stream(stream))
    _check(code, "hs2_full_attn_select")
    return out, idx, lse


def full_attn_select_blocks(q: torch.Tensor, cache: Cache, window: int = 128, k_sel: int = 1024,
                            block: int = 64, sm_scale: Optional[float] = None,
                            workspace: Optional[torch.Tensor] = None,
                            out: Optional[torch.Tensor] = None, idx: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                            stream=None):
    """Full-attention layer + block-level selection (whole blocks of ``block``
    positions, the first-generation comparator).  Returns (out, idx, lse)."""
    n_q, h = _check_q(q, cache)
    B = cache.batch
    sm_scale = default_scale() if sm_scale is None else sm_scale
    if workspace is None:
        workspace = alloc_workspace(cache, n_q, h, window, k_sel)
    if out is None:
        out = torch.empty(B, n_q, h, 128, dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty(B, n_q, window + k_sel, dtype=torch.int32, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(B, n_q, h, dtype=torch.float32, device=q.device)
    code = lib().hs2_full_attn_select_blocks(q.data_ptr(), n_q, h, cache.ref(), window, k_sel,
                                             block, sm_scale, out.data_ptr(), idx.data_ptr(),
                                             _ptr(lse), workspace.data_ptr(), workspace.numel(),
                                             _stream(stream))
    _check(code, "hs2_full_attn_select_blocks")
    return out, idx, lse


def select_blocks(q, cache: Cache, workspace: torch.Tensor, window=128, k_sel=1024, block=64,
                  sm_scale=None, idx=None, stream=None):
    """Block-level selection alone; must follow full_attn on the same workspace."""
    n_q, h = _check_q(q, cache)
    sm_scale = default_scale() if sm_scale is None else sm_scale
    if idx is None:
        idx = torch.empty(cache.batch, n_q, window + k_sel, dtype=torch.int32, device=q.device)
    code = lib().hs2_select_blocks(q.data_ptr(), n_q, h, cache.ref(), window, k_sel, block,
                                   sm_scale, idx.data_ptr(), workspace.data_ptr(),
                                   workspace.numel(), _stream(stream))
    _check(code, "hs2_select_blocks")
    return idx


def prefill_workspace(cache: Cache, n_q: int, h_q: int, device=None) -> torch.Tensor:
    """A zero-filled workspace (uint8 tensor) for prefill_attn at these sizes."""
    n = lib().hs2_prefill_workspace_bytes(cache.batch, n_q, h_q, cache.max_len, cache.dtype)
    if n == 0:
        raise Hs2Error(2, "hs2_prefill_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or cache.k.device)


def prefill_attn(q: torch.Tensor, cache: Cache, sm_scale: Optional[float] = None,
                 workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, want_lse: bool = True, stream=None):
    """Full-attention layer over a chunk of n_q new tokens per sequence (chunked
    prefill; no selection).  Returns (out, lse)."""
    n_q, h = _check_q(q, cache)
    sm_scale = default_scale() if sm_scale is None else sm_scale
    if workspace is None:
        workspace = prefill_workspace(cache, n_q, h)
    if out is None:
        out = torch.empty(cache.batch, n_q, h, 128, dtype=torch.float32, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty(cache.batch, n_q, h, dtype=torch.float32, device=q.device)
    code = lib().hs2_prefill_attn(q.data_ptr(), n_q, h, cache.ref(), sm_scale, out.data_ptr(),
                                  _ptr(lse), workspace.data_ptr(), workspace.numel(),
                                  _stream(stream))
    _check(code, "hs2_prefill_attn")
    return out, lse


def full_attn(q, cache: Cache, window=128, k_sel=1024, sm_scale=None, workspace=None,
              out=None, lse=None, stream=None):
    """Full-attention layer alone (leaves the per-head lse in the workspace)."""
    n_q, h = _check_q(q, cache)
    sm_scale = default_scale() if sm_scale is None else sm_scale
    if workspace is None:
        workspace = alloc_workspace(cache, n_q, h, window, k_sel)
    if out is None:
        out = torch.empty(cache.batch, n_q, h, 128, dtype=torch.float32, device=q.device)
    code = lib().hs2_full_attn(q.data_ptr(), n_q, h, cache.ref(), window, k_sel, sm_scale,
                               out.data_ptr(), _ptr(lse), workspace.data_ptr(),
                               workspace.numel(), _stream(stream))
    _check(code, "hs2_full_attn")
    return out


def select(q, cache: Cache, workspace: torch.Tensor, window=128, k_sel=1024, sm_scale=None,
           idx=None, stream=None):
    """Token selection alone; must follow full_attn on the same workspace."""
    n_q, h = _check_q(q, cache)
    sm_scale = default_scale() if sm_scale is None else sm_scale
    if idx is None:
        idx = torch.empty(cache.batch, n_q, window + k_sel, dtype=torch.int32, device=q.device)
    code = lib().hs2_select(q.data_ptr(), n_q, h, cache.ref(), window, k_sel, sm_scale,
                            idx.data_ptr(), workspace.data_ptr(), workspace.numel(),
                            _stream(stream))
    _check(code, "hs2_select")
    return idx


def sparse_attn(q_layer: torch.Tensor, cache: Cache, idx: torch.Tensor,
                workspace: torch.Tensor, sm_scale: Optional[float] = None,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One reusing sparse-attention layer over the rows named by ``idx``."""
    n_q, h = _check_q(q_layer, cache)
    if idx.dtype != torch.int32 or not idx.is_contiguous() or idx.dim() != 3 \
            or idx.shape[:2] != (cache.batch, n_q):
        raise ValueError("idx must be contiguous int32 [B, n_q, width]")
    sm_scale = default_scale() if sm_scale is None else sm_scale
    if out is None:
        out = torch.empty(cache.batch, n_q, h, 128, dtype=torch.float32, device=q_layer.device)
    code = lib().hs2_sparse_attn(q_layer.data_ptr(), n_q, h, cache.ref(), idx.data_ptr(),
                                 idx.shape[2], sm_scale, out.data_ptr(), workspace.data_ptr(),
                                 workspace.numel(), _stream(stream))
    _check(code, "hs2_sparse_attn")
    return out


def kv_append(k_new: torch.Tensor, v_new: torch.Tensor, cache: Cache, workspace: torch.Tensor,
              stream=None) -> None:
    """Appends n_new tokens per sequence to ``cache`` (bf16 [B, n_new, 128] keys and
    values; FP8 caches quantise each new row with its own scale) and grows
    ``cache.lens`` in place."""
    for name, t in (("k_new", k_new), ("v_new", v_new)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous() or t.dim() != 3 \
                or t.shape[0] != cache.batch or t.shape[2] != 128:
            raise ValueError(f"{name} must be contiguous bf16 [B, n_new, 128] on the device")
    if k_new.shape != v_new.shape:
        raise ValueError("k_new and v_new must have the same shape")
    code = lib().hs2_kv_append(k_new.data_ptr(), v_new.data_ptr(), k_new.shape[1], cache.ref(),
                               cache.lens.data_ptr(), workspace.data_ptr(), workspace.numel(),
                               _stream(stream))
    _check(code, "hs2_kv_append")


def check_device_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, return (and clear) the first device-side error code (0 = none)."""
    return lib().hs2_check_device_status(workspace.data_ptr(), _stream(stream))
