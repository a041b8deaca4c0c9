"""Seeded synthetic inputs for the hybrid-block decode step.

This module only draws random tensors and lays them out; it holds none of the
method's arithmetic (no attention, no importance, no selection).  Both the CUDA
path (through the binding) and the float64 oracle consume what it returns.

Recipe (the same for every workload):
  * one ``torch.Generator`` per tensor family, seeded from the workload seed,
    so that adding a sparse layer does not change the cache or the queries;
  * queries, keys and values are N(0, 1) float32 draws, rounded once to bf16
    (round-to-nearest-even) or, for the FP8 cache, clamped to +-448 and rounded
    to OCP E4M3 ("fn") codes; FP8 rows carry a per-token float32 scale drawn
    U[0.5, 2] for K and for V;
  * rows past ``lens[b]`` hold NaN (bf16 NaN, E4M3 code 0x7F, NaN scale), so
    any read beyond a sequence's length poisons the result;
  * planted needles: key ``j`` is replaced by ``delta / (sm_scale * |q_h|^2) * q_h``
    for head ``h = needle_number mod h_q`` of the full layer's last query token,
    which gives that head the logit ``delta`` before the key is rounded.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import torch

HEAD_DIM = 128
E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and structure of one synthetic decode (or append) step."""

    name: str
    batch: int
    max_len: int
    n_q: int
    h_q: int
    kv: str                      # "bf16" or "fp8"
    n_sparse: int                # reusing sparse layers in the hybrid block
    seed: int
    len_lo: Optional[int] = None  # ragged lengths: U[len_lo, max_len]; None = all max_len
    n_needles: int = 0
    needle_layout: str = "none"  # "uniform" | "even" | "loguniform" | "none"
    needle_delta: float = 4.0
    window: int = 128
    k_sel: int = 1024


# The five workloads of the hybrid-block decode step (window 128 + top-1024).
WORKLOADS = {
    1: Workload("decode b1 ctx4096 bf16 h16", batch=1, max_len=4096, n_q=1, h_q=16,
                kv="bf16", n_sparse=3, seed=1001, n_needles=8,
                needle_layout="uniform", needle_delta=4.0),
    2: Workload("decode b8 ctx131072 bf16 h16", batch=8, max_len=131072, n_q=1, h_q=16,
                kv="bf16", n_sparse=3, seed=1002, n_needles=64,
                needle_layout="even", needle_delta=4.0),
    3: Workload("decode b4 ctx204800-262144 fp8 h16", batch=4, max_len=262144, n_q=1,
                h_q=16, kv="fp8", n_sparse=5, seed=1003, len_lo=204800),
    # FP8 per-token scales U[0.5, 2] widen the logit spread, so the top-1024 of 2^20
    # keys x 64 heads starts near logit 7.3; needles get logit 10 to clear it.
    4: Workload("decode b1 ctx1048576 fp8 h64", batch=1, max_len=1048576, n_q=1, h_q=64,
                kv="fp8", n_sparse=3, seed=1004, n_needles=256,
                needle_layout="loguniform", needle_delta=10.0),
    5: Workload("append 64x16 ctx131072 bf16", batch=1, max_len=131072, n_q=64, h_q=16,
                kv="bf16", n_sparse=3, seed=1005),
}


@dataclasses.dataclass
class Inputs:
    """Host (CPU) tensors of one step; ``k``/``v`` are bf16 or uint8 E4M3 codes."""

    q: torch.Tensor                    # bf16 [B, n_q, h_q, 128]
    q_layers: List[torch.Tensor]       # bf16 [B, n_q, h_q, 128] per sparse layer
    k: torch.Tensor                    # bf16 or uint8 [B, max_len, 128]
    v: torch.Tensor
    k_scale: Optional[torch.Tensor]    # fp32 [B, max_len] (FP8 only)
    v_scale: Optional[torch.Tensor]
    lens: torch.Tensor                 # int32 [B]
    sm_scale: float                    # exactly representable in fp32
    window: int
    k_sel: int
    kv: str
    needles: List[List[Tuple[int, int]]]  # per sequence: (position, head)

    @property
    def batch(self) -> int:
        return self.k.shape[0]

    @property
    def max_len(self) -> int:
        return self.k.shape[1]

    @property
    def n_q(self) -> int:
        return self.q.shape[1]

    @property
    def h_q(self) -> int:
        return self.q.shape[2]


def fp32(x: float) -> float:
    """The float32 value nearest to ``x``, as a Python float."""
    return float(torch.tensor(x, dtype=torch.float32).item())


def default_sm_scale(head_dim: int = HEAD_DIM) -> float:
    return fp32(1.0 / math.sqrt(head_dim))


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator()
    g.manual_seed(seed)
    return g


def to_e4m3_codes(x: torch.Tensor) -> torch.Tensor:
    """Round float32 values to OCP E4M3 codes (nearest-even, saturating at +-448)."""
    return x.clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn).view(torch.uint8)


def _needle_positions(layout: str, n: int, length: int, window: int,
                      g: torch.Generator) -> List[int]:
    hi = length - window          # needles sit outside the forced window
    if n <= 0 or hi <= 0:
        return []
    if layout == "uniform":
        pos = torch.randperm(hi, generator=g)[:n].tolist()
    elif layout == "even":
        pos = [(i * hi) // n for i in range(n)]
    elif layout == "loguniform":
        lo_d, hi_d = math.log(window + 1), math.log(length)
        u = torch.rand(n, generator=g, dtype=torch.float64).tolist()
        pos = [length - int(round(math.exp(lo_d + (hi_d - lo_d) * x))) for x in u]
        pos = [min(max(p, 0), hi - 1) for p in pos]
    else:
        raise ValueError(f"unknown needle layout {layout!r}")
    seen, out = set(), []
    for p in pos:
        if p not in seen:
            seen.add(p)
            out.append(p)
    return sorted(out)


def make_inputs(batch: int, max_len: int, n_q: int, h_q: int, kv: str = "bf16",
                n_sparse: int = 1, seed: int = 0, lens: Optional[Sequence[int]] = None,
                window: int = 128, k_sel: int = 1024, n_needles: int = 0,
                needle_layout: str = "none", needle_delta: float = 4.0,
                q_zero: bool = False, identical_keys: bool = False,
                sm_scale: Optional[float] = None) -> Inputs:
    """Draw one step's inputs.  ``lens`` defaults to ``max_len`` for every row."""
    if kv not in ("bf16", "fp8"):
        raise ValueError("kv must be 'bf16' or 'fp8'")
    d = HEAD_DIM
    sm_scale = default_sm_scale(d) if sm_scale is None else fp32(sm_scale)
    base = seed * 1000
    q32 = torch.randn(batch, n_q, h_q, d, generator=_gen(base + 1))
    if q_zero:
        q32.zero_()
    q = q32.to(torch.bfloat16)
    q_layers = [torch.randn(batch, n_q, h_q, d, generator=_gen(base + 10 + i)).to(torch.bfloat16)
                for i in range(n_sparse)]
    if lens is None:
        lens_t = torch.full((batch,), max_len, dtype=torch.int32)
    else:
        lens_t = torch.tensor(list(lens), dtype=torch.int32)
    gk, gv, gs = _gen(base + 100), _gen(base + 200), _gen(base + 300)
    gn = _gen(base + 400)
    fp8 = kv == "fp8"
    kdt = torch.uint8 if fp8 else torch.bfloat16
    k = torch.empty(batch, max_len, d, dtype=kdt)
    v = torch.empty(batch, max_len, d, dtype=kdt)
    k_scale = torch.empty(batch, max_len, dtype=torch.float32) if fp8 else None
    v_scale = torch.empty(batch, max_len, dtype=torch.float32) if fp8 else None
    needles: List[List[Tuple[int, int]]] = []
    for b in range(batch):
        L = int(lens_t[b])
        kb = torch.randn(max_len, d, generator=gk)
        vb = torch.randn(max_len, d, generator=gv)
        if identical_keys:
            kb[:] = kb[0]
        if fp8:
            ks = torch.rand(max_len, generator=gs) * 1.5 + 0.5
            vs = torch.rand(max_len, generator=gs) * 1.5 + 0.5
        nb = []
        for i, pos in enumerate(_needle_positions(needle_layout, n_needles, L, window, gn)):
            h = i % h_q
            qh = q[b, n_q - 1, h].to(torch.float64)
            kn = (needle_delta / (sm_scale * float(qh.dot(qh)))) * qh
            if fp8:
                kb[pos] = (kn / float(ks[pos])).to(torch.float32)
            else:
                kb[pos] = kn.to(torch.float32)
            nb.append((pos, h))
        needles.append(nb)
        if fp8:
            kc, vc = to_e4m3_codes(kb), to_e4m3_codes(vb)
            kc[L:] = 0x7F
            vc[L:] = 0x7F
            ks[L:] = float("nan")
            vs[L:] = float("nan")
            k[b], v[b] = kc, vc
            k_scale[b], v_scale[b] = ks, vs
        else:
            kb, vb = kb.to(torch.bfloat16), vb.to(torch.bfloat16)
            kb[L:] = float("nan")
            vb[L:] = float("nan")
            k[b], v[b] = kb, vb
    return Inputs(q=q, q_layers=q_layers, k=k, v=v, k_scale=k_scale, v_scale=v_scale,
                  lens=lens_t, sm_scale=sm_scale, window=window, k_sel=k_sel, kv=kv,
                  needles=needles)


def generate(workload: Workload) -> Inputs:
    """Inputs of one of the named workloads (deterministic in ``workload.seed``)."""
    lens = None
    if workload.len_lo is not None:
        lens = torch.randint(workload.len_lo, workload.max_len + 1, (workload.batch,),
                             generator=_gen(workload.seed * 1000 + 500)).tolist()
    return make_inputs(workload.batch, workload.max_len, workload.n_q, workload.h_q,
                       kv=workload.kv, n_sparse=workload.n_sparse, seed=workload.seed,
                       lens=lens, window=workload.window, k_sel=workload.k_sel,
                       n_needles=workload.n_needles, needle_layout=workload.needle_layout,
                       needle_delta=workload.needle_delta)


def numpy_bits(inp: Inputs) -> dict:
    """The raw storage of ``inp`` as numpy arrays (bf16 -> uint16 bits, E4M3 -> uint8 codes)."""
    def bits(t: torch.Tensor):
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view("uint16")
        return t.numpy()
    return dict(
        q=bits(inp.q), q_layers=[bits(x) for x in inp.q_layers], k=bits(inp.k), v=bits(inp.v),
        k_scale=None if inp.k_scale is None else inp.k_scale.numpy(),
        v_scale=None if inp.v_scale is None else inp.v_scale.numpy(),
        lens=inp.lens.numpy(), sm_scale=inp.sm_scale, window=inp.window, k_sel=inp.k_sel,
        kv=inp.kv)
