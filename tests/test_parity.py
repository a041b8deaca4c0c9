"""GPU parity: libhs2 (through its C ABI) against the float64 oracle.

Index sets must equal the oracle's except inside the tie band (gap between the
k-th and (k+1)-th importance below 1e-6 relative); outputs within max-abs 2e-3
(bf16 cache) or 1e-2 (FP8 cache); lse within 1e-4, and the float64 lse that the
selection uses within 1e-6.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from long_context_token_b200 import hs2, workloads
from _util import check_block_index_set, check_index_set

pytestmark = [pytest.mark.gpu, pytest.mark.filterwarnings("ignore::RuntimeWarning")]

TOL = {"bf16": 2e-3, "fp8": 1e-2}
LSE_TOL = 1e-4
LSE64_TOL = 1e-6
# The CUDA-core full layer (shapes the tensor-core kernels do not take) sums each logit's
# 128 products in float32 one after another: about 2^-24 x 128 of sum |q_c k_c| of
# rounding, which over the 128 heads of a row reaches about 1.2e-6 in the lse.
LSE64_TOL_CUDA_CORE = 2e-6


def cuda_core_path(kv: str, n_q: int, h: int) -> bool:
    """Shapes whose full layer runs on the CUDA-core kernel: FP8 with more than 64 heads,
    bf16 with 80, 96 or 112 heads."""
    return (kv == "fp8" and h > 64) or (kv == "bf16" and h in (80, 96, 112))


def run_gpu(inp: workloads.Inputs, twice: bool = False):
    dev = torch.device("cuda:0")
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev),
                      None if inp.k_scale is None else inp.k_scale.to(dev),
                      None if inp.v_scale is None else inp.v_scale.to(dev))
    q = inp.q.to(dev)
    ws = hs2.alloc_workspace(cache, inp.n_q, inp.h_q, inp.window, inp.k_sel)
    runs = []
    for _ in range(2 if twice else 1):
        out, idx, lse = hs2.full_attn_select(q, cache, inp.window, inp.k_sel, inp.sm_scale, ws)
        lse64 = hs2.workspace_lse64(ws, cache, inp.n_q, inp.h_q, inp.window, inp.k_sel)
        lse64 = lse64.cpu().numpy()  # before the sparse layers reuse the workspace
        sp = [hs2.sparse_attn(ql.to(dev), cache, idx, ws, inp.sm_scale) for ql in inp.q_layers]
        torch.cuda.synchronize()
        runs.append(dict(out=out.cpu().numpy(), idx=idx.cpu().numpy(), lse=lse.cpu().numpy(),
                         lse64=lse64, sparse=[s.cpu().numpy() for s in sp]))
    status = hs2.check_device_status(ws)
    return runs, status


def compare(inp: workloads.Inputs, res: dict, sparse_full: bool = True):
    return compare_bits(workloads.numpy_bits(inp), res, sparse_full)


def compare_bits(bits: dict, res: dict, sparse_full: bool = True):
    """Checks one GPU step against the oracle run on the cache ``bits``."""
    ref = oracle.full_attn_select(bits, keep_importance=True)
    tol = TOL[bits["kv"]]
    err = np.abs(res["out"] - ref["out"]).max()
    assert err < tol, f"full-layer output max-abs error {err}"
    lerr = np.abs(res["lse"] - ref["lse"]).max()
    assert lerr < LSE_TOL, f"lse error {lerr}"
    if "lse64" in res:
        # The float64 lse that the selection shifts each head's scores by: its error moves
        # the ranking directly, so it is held to the selection's tie band.
        B, n_q, h = ref["lse"].shape
        tol64 = LSE64_TOL_CUDA_CORE if cuda_core_path(bits["kv"], n_q, h) else LSE64_TOL
        l64 = np.abs(res["lse64"].reshape(ref["lse"].shape) - ref["lse"]).max()
        assert l64 <= tol64, f"float64 lse error {l64}"
    B, n_q = bits["q"].shape[:2]
    window, k_sel = bits["window"], bits["k_sel"]
    n_exact = 0
    for b in range(B):
        L = int(bits["lens"][b])
        for i in range(n_q):
            p = L - n_q + i
            msg = check_index_set(res["idx"][b, i], ref["idx"][b, i], ref["imp"][b * n_q + i],
                                  p, window, k_sel)
            assert msg is None, f"(b={b}, i={i}, p={p}): {msg}"
            n_exact += int(np.array_equal(res["idx"][b, i], ref["idx"][b, i]))
    # Sparse layers: fed the GPU's own index set (identical to the oracle's outside
    # the tie band), compared with the oracle's sparse layer on that set.
    for li, ql in enumerate(bits["q_layers"]):
        want = oracle.sparse_attn(bits, ql, res["idx"] if sparse_full else ref["idx"])
        e = np.abs(res["sparse"][li] - want).max()
        assert e < tol, f"sparse layer {li} max-abs error {e}"
    return n_exact


SMALL = [
    dict(id="b1-L4096-h16-bf16", batch=1, max_len=4096, n_q=1, h_q=16, kv="bf16", seed=101,
         n_needles=8, needle_layout="uniform"),
    dict(id="ragged-b3-bf16", batch=3, max_len=5000, n_q=1, h_q=16, kv="bf16", seed=102,
         lens=[5000, 1200, 1153]),
    dict(id="short-contexts", batch=5, max_len=1300, n_q=1, h_q=16, kv="bf16", seed=103,
         lens=[1, 100, 128, 1152, 1153]),
    dict(id="h64-fp8-ragged", batch=2, max_len=3000, n_q=1, h_q=64, kv="fp8", seed=104,
         lens=[3000, 2901]),
    dict(id="h32-append4", batch=1, max_len=2500, n_q=4, h_q=32, kv="bf16", seed=105),
    dict(id="h128-bf16", batch=1, max_len=2000, n_q=1, h_q=128, kv="bf16", seed=106),
    dict(id="h48-fp8", batch=2, max_len=1800, n_q=2, h_q=48, kv="fp8", seed=107,
         lens=[1800, 1500]),
    dict(id="tiny-window4-k8", batch=2, max_len=48, n_q=3, h_q=16, kv="bf16", seed=108,
         lens=[48, 13], window=4, k_sel=8),
    dict(id="window1-k1", batch=1, max_len=300, n_q=2, h_q=16, kv="fp8", seed=109,
         window=1, k_sel=1),
    dict(id="max-width-4096", batch=1, max_len=10000, n_q=1, h_q=16, kv="bf16", seed=110,
         window=128, k_sel=3968),
    dict(id="append64-fp8", batch=1, max_len=3000, n_q=64, h_q=16, kv="fp8", seed=111),
    dict(id="ragged-tail-fp8", batch=3, max_len=9000, n_q=1, h_q=16, kv="fp8", seed=112,
         lens=[8999, 4097, 1333]),
    # several new tokens per sequence (bf16): 128 query rows per CTA, groups of 128 / h
    # tokens, the last group partial; contexts whose chunks end inside a 64-key tile
    dict(id="append13-h16-ragged", batch=2, max_len=7000, n_q=13, h_q=16, kv="bf16",
         seed=113, lens=[7000, 2222]),
    dict(id="append5-h48", batch=1, max_len=4321, n_q=5, h_q=48, kv="bf16", seed=114),
    dict(id="append3-h64-short", batch=2, max_len=700, n_q=3, h_q=64, kv="bf16", seed=115,
         lens=[700, 130]),
    # several tokens on an FP8 cache whose rows are an odd number of keys long (the row
    # buffers of the fused selection are padded to keep their 16-byte copies aligned)
    dict(id="append3-fp8-odd-len", batch=2, max_len=1509, n_q=3, h_q=16, kv="fp8", seed=116,
         lens=[1509, 1402]),
    dict(id="append2-fp8-h64-odd", batch=3, max_len=2001, n_q=2, h_q=64, kv="fp8", seed=117,
         lens=[2001, 1999, 1200]),
    # shapes served by the CUDA-core kernels: FP8 with more than 64 heads, bf16 with 80,
    # 96 or 112 heads
    dict(id="h128-fp8-cuda-core", batch=2, max_len=2500, n_q=1, h_q=128, kv="fp8", seed=118,
         lens=[2500, 1777]),
    dict(id="h96-fp8-append2-cuda-core", batch=1, max_len=1900, n_q=2, h_q=96, kv="fp8",
         seed=119),
    dict(id="h80-bf16-cuda-core", batch=2, max_len=3000, n_q=1, h_q=80, kv="bf16", seed=120,
         lens=[3000, 2111]),
    dict(id="h112-bf16-cuda-core", batch=1, max_len=2300, n_q=1, h_q=112, kv="bf16", seed=121),
    dict(id="h96-bf16-append3-cuda-core", batch=2, max_len=1700, n_q=3, h_q=96, kv="bf16",
         seed=122, lens=[1700, 1234]),
]


def test_long_chunks_in_several_pieces_match_oracle():
    """74 sequences of up to 32768 keys: two CTAs a row, so each CTA's chunk (16384 keys)
    is longer than the on-chip piece of the fused selection's bounds, and the candidates
    of a chunk are kept in the row's candidate buffer instead of on chip."""
    lens = [32768 - 37 * i for i in range(74)]
    inp = workloads.make_inputs(74, 32768, n_q=1, h_q=16, kv="bf16", seed=125, lens=lens,
                                n_sparse=1)
    runs, status = run_gpu(inp)
    assert status == 0
    compare(inp, runs[0])


def test_long_chunks_with_all_keys_tied_match_oracle():
    """A zero query over long chunks: every key of a row ties, so the whole row is the band
    -- each CTA re-scores its ~16000 band keys in rounds of at most 512 on chip, and the
    band is ranked by the radix fallback; the lowest positions win the ties."""
    lens = [32768 - 37 * i for i in range(74)]
    inp = workloads.make_inputs(74, 32768, n_q=1, h_q=16, kv="bf16", seed=126, lens=lens,
                                n_sparse=1, q_zero=True)
    runs, status = run_gpu(inp)
    assert status == 0
    compare(inp, runs[0])


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c["id"])
def test_small_cases_match_oracle(case):
    kw = {k: v for k, v in case.items() if k != "id"}
    inp = workloads.make_inputs(n_sparse=2, **kw)
    runs, status = run_gpu(inp)
    assert status == 0
    compare(inp, runs[0])


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_zero_query_ties_pick_lowest_positions(kv):
    inp = workloads.make_inputs(2, 20000, n_q=1, h_q=16, kv=kv, seed=120, q_zero=True,
                                lens=[20000, 7000])
    runs, status = run_gpu(inp)
    assert status == 0
    for b, L in enumerate([20000, 7000]):
        want = np.concatenate([np.arange(1024), np.arange(L - 128, L)])
        assert np.array_equal(runs[0]["idx"][b, 0], want)
    compare(inp, runs[0])


def test_identical_keys_are_all_ties():
    inp = workloads.make_inputs(1, 6000, n_q=2, h_q=16, seed=121, identical_keys=True)
    runs, status = run_gpu(inp)
    assert status == 0
    for i in range(2):
        p = 6000 - 2 + i
        want = np.concatenate([np.arange(1024), np.arange(p - 127, p + 1)])
        assert np.array_equal(runs[0]["idx"][0, i], want)
    compare(inp, runs[0])


# 2 x 60000 keys: 67 CTAs a row, about 7 of the row's 469 tiles each, so that the default mode
# claims tiles at run time (CTA r starts with tiles r, r + S, ... and claims the rest).
REPEAT_CASES = [dict(kv="fp8", seed=122), dict(kv="bf16", seed=123)]


@pytest.mark.parametrize("case", REPEAT_CASES, ids=lambda c: c["kv"])
def test_repeat_runs_are_bitwise_identical_in_deterministic_mode(case):
    inp = workloads.make_inputs(2, 60000, n_q=1, h_q=16, kv=case["kv"], seed=case["seed"],
                                n_sparse=1, lens=[60000, 47111])
    hs2.set_deterministic(True)
    try:
        runs = [run_gpu(inp, twice=True)[0] for _ in range(3)]
    finally:
        hs2.set_deterministic(False)
    a = runs[0][0]
    for b in [r for pair in runs for r in pair][1:]:
        assert np.array_equal(a["idx"], b["idx"])
        assert np.array_equal(a["out"], b["out"]) and np.array_equal(a["lse"], b["lse"])
        assert np.array_equal(a["sparse"][0], b["sparse"][0])
    compare(inp, a)


@pytest.mark.parametrize("case", REPEAT_CASES, ids=lambda c: c["kv"])
def test_repeat_runs_agree_within_rounding_by_default(case):
    """Run-time tile sharing regroups the float32 partial sums between runs: the index set
    stays the same (no key of these inputs sits within the lse's rounding of another) and
    the outputs differ by rounding only -- for an FP8 cache also by the E4M3 split of P,
    whose power-of-two scale follows the largest V scale among the tiles a CTA took
    (values of P v_scale below 2^-6 of it are kept to 2^-18): far inside the 1e-2
    tolerance, above float32 rounding."""
    out_tol = 1e-6 if case["kv"] == "bf16" else 1e-4
    inp = workloads.make_inputs(2, 60000, n_q=1, h_q=16, kv=case["kv"], seed=case["seed"],
                                n_sparse=1, lens=[60000, 47111])
    runs = [r for _ in range(3) for r in run_gpu(inp, twice=True)[0]]
    a = runs[0]
    for b in runs[1:]:
        assert np.array_equal(a["idx"], b["idx"])
        assert np.abs(a["out"] - b["out"]).max() <= out_tol
        assert np.abs(a["lse64"] - b["lse64"]).max() <= 1e-6
        assert np.abs(a["sparse"][0] - b["sparse"][0]).max() <= out_tol
    compare(inp, a)


def test_device_status_reports_bad_index_and_length():
    dev = torch.device("cuda:0")
    inp = workloads.make_inputs(2, 600, n_q=1, h_q=16, seed=123, lens=[600, 300])
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev))
    ws = hs2.alloc_workspace(cache, 1, 16)
    idx = torch.full((2, 1, 8), -1, dtype=torch.int32, device=dev)
    idx[0, 0, :3] = torch.tensor([0, 5, 599])
    idx[1, 0, 0] = 300                     # == lens[1]: out of range
    hs2.sparse_attn(inp.q.to(dev), cache, idx, ws)
    assert hs2.check_device_status(ws) == 6
    assert hs2.check_device_status(ws) == 0          # cleared by the read
    bad = hs2.Cache(inp.k.to(dev), inp.v.to(dev), torch.tensor([601, 300], dtype=torch.int32,
                                                                device=dev))
    hs2.full_attn_select(inp.q.to(dev), bad, workspace=ws)
    assert hs2.check_device_status(ws) == 7


def test_sparse_layer_skips_padding_and_empty_rows():
    dev = torch.device("cuda:0")
    inp = workloads.make_inputs(1, 500, n_q=2, h_q=16, seed=124, n_sparse=1)
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev))
    ws = hs2.alloc_workspace(cache, 2, 16)
    idx = torch.full((1, 2, 300), -1, dtype=torch.int32, device=dev)
    idx[0, 0, 7:200] = torch.arange(100, 293, dtype=torch.int32)
    out = hs2.sparse_attn(inp.q_layers[0].to(dev), cache, idx, ws).cpu().numpy()
    assert hs2.check_device_status(ws) == 0
    bits = workloads.numpy_bits(inp)
    want = oracle.sparse_attn(bits, bits["q_layers"][0][:, :1], idx[:, :1].cpu().numpy())
    assert np.abs(out[:, :1] - want).max() < 2e-3
    assert np.all(out[0, 1] == 0.0)          # an empty index row yields zeros


@pytest.mark.parametrize("kv,h_q", [("bf16", 16), ("fp8", 64), ("bf16", 48)])
@pytest.mark.parametrize("width", [1, 127, 129, 1152, 2049, 4096])
def test_sparse_layer_widths(kv, h_q, width):
    """Index rows of 1 to 32 tiles (one to several tiles per CTA of the merging
    cluster), with padding slots and a row whose only valid entry is its last."""
    dev = torch.device("cuda:0")
    inp = workloads.make_inputs(2, 6000, n_q=2, h_q=h_q, kv=kv, seed=131 + width, n_sparse=1,
                                lens=[6000, 4500])
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev),
                      None if inp.k_scale is None else inp.k_scale.to(dev),
                      None if inp.v_scale is None else inp.v_scale.to(dev))
    ws = hs2.alloc_workspace(cache, 2, h_q)
    rng = np.random.default_rng(width)
    idx = np.full((2, 2, width), -1, dtype=np.int32)
    for b in range(2):
        L = int(inp.lens[b])
        for i in range(2):
            n = width if (b, i) != (1, 1) else 1
            pos = np.sort(rng.choice(L - 1, size=n, replace=False)).astype(np.int32)
            if n == width and width > 4:
                pos[rng.choice(width, size=width // 5, replace=False)] = -1   # padding slots
            if n == 1:
                idx[b, i, -1] = pos[0]
            else:
                idx[b, i] = pos
    idx_t = torch.from_numpy(idx).to(dev)
    out = hs2.sparse_attn(inp.q_layers[0].to(dev), cache, idx_t, ws, inp.sm_scale).cpu().numpy()
    assert hs2.check_device_status(ws) == 0
    bits = workloads.numpy_bits(inp)
    want = oracle.sparse_attn(bits, bits["q_layers"][0], idx)
    err = np.abs(out - want).max()
    assert err < TOL[kv], f"max-abs error {err}"


@pytest.mark.slow
@pytest.mark.parametrize("n", sorted(workloads.WORKLOADS))
def test_full_size_workloads_match_oracle(n):
    w = workloads.WORKLOADS[n]
    inp = workloads.generate(w)
    runs, status = run_gpu(inp)
    assert status == 0
    compare(inp, runs[0])
    idx = runs[0]["idx"]
    for b, needles in enumerate(inp.needles):
        for pos, _ in needles:
            assert pos in idx[b, w.n_q - 1], f"needle at {pos} not selected"


# A decode loop: every step appends n_new tokens per sequence (the new tokens' K/V),
# then runs the full layer with selection and the sparse layers for those tokens as
# queries.  Sequence 1 starts empty; sequence 0 ends exactly at max_len.
DECODE_LOOP = [
    dict(id="bf16-h16", kv="bf16", h_q=16, n_new=1, seed=141),
    dict(id="fp8-h16", kv="fp8", h_q=16, n_new=1, seed=142),
    dict(id="fp8-h64", kv="fp8", h_q=64, n_new=1, seed=143),
    dict(id="fp8-h16-append3", kv="fp8", h_q=16, n_new=3, seed=144),
    dict(id="bf16-h32-append4", kv="bf16", h_q=32, n_new=4, seed=145),
]
LOOP_STEPS = 3


def _new_rows(gen: torch.Generator, batch: int, n_new: int) -> torch.Tensor:
    """bf16 [B, n_new, 128]: Gaussian rows with per-token magnitudes spread over
    e^[-3, 1], one all-zero row (scale 1) and one row of tiny entries under a
    dominant +5 / -6 pair (its other codes fall into the E4M3 subnormals)."""
    x = torch.randn(batch, n_new, 128, generator=gen)
    x *= torch.exp(torch.rand(batch, n_new, 1, generator=gen) * 4 - 3)
    x[0, 0] = 0
    x[-1, -1] *= 1e-4
    x[-1, -1, 7], x[-1, -1, 9] = 5.0, -6.0
    return x.to(torch.bfloat16)


def _bits_of(t: torch.Tensor) -> np.ndarray:
    t = t.cpu()
    return (t.view(torch.int16).numpy().view("uint16") if t.dtype == torch.bfloat16
            else t.numpy())


def _assert_cache_equal(cache: hs2.Cache, want: dict):
    assert np.array_equal(cache.lens.cpu().numpy(), want["lens"])
    assert np.array_equal(_bits_of(cache.k), want["k"]), "K rows differ"
    assert np.array_equal(_bits_of(cache.v), want["v"]), "V rows differ"
    if want["kv"] == "fp8":
        for name in ("k_scale", "v_scale"):
            got = getattr(cache, name).cpu().numpy().view(np.uint32)
            assert np.array_equal(got, want[name].view(np.uint32)), f"{name} differs"


@pytest.mark.parametrize("case", DECODE_LOOP, ids=lambda c: c["id"])
def test_decode_loop_with_append_matches_oracle(case):
    dev = torch.device("cuda:0")
    n_new, h_q = case["n_new"], case["h_q"]
    lens0 = [1500, 0]
    max_len = lens0[0] + LOOP_STEPS * n_new
    inp = workloads.make_inputs(2, max_len, n_q=n_new, h_q=h_q, kv=case["kv"],
                                seed=case["seed"], lens=lens0, n_sparse=2)
    bits = workloads.numpy_bits(inp)
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev),
                      None if inp.k_scale is None else inp.k_scale.to(dev),
                      None if inp.v_scale is None else inp.v_scale.to(dev))
    ws = hs2.alloc_workspace(cache, n_new, h_q)
    gen = torch.Generator().manual_seed(case["seed"])
    for step in range(LOOP_STEPS):
        k_new, v_new = _new_rows(gen, 2, n_new), _new_rows(gen, 2, n_new)
        hs2.kv_append(k_new.to(dev), v_new.to(dev), cache, ws)
        bits = oracle.kv_append(bits, _bits_of(k_new), _bits_of(v_new))
        q = torch.randn(2, n_new, h_q, 128, generator=gen).to(torch.bfloat16)
        q_layers = [torch.randn(2, n_new, h_q, 128, generator=gen).to(torch.bfloat16)
                    for _ in range(2)]
        out, idx, lse = hs2.full_attn_select(q.to(dev), cache, inp.window, inp.k_sel,
                                             inp.sm_scale, ws)
        sp = [hs2.sparse_attn(ql.to(dev), cache, idx, ws, inp.sm_scale) for ql in q_layers]
        assert hs2.check_device_status(ws) == 0, f"step {step}"
        _assert_cache_equal(cache, bits)
        bits = dict(bits, q=_bits_of(q), q_layers=[_bits_of(x) for x in q_layers])
        compare_bits(bits, dict(out=out.cpu().numpy(), idx=idx.cpu().numpy(),
                                lse=lse.cpu().numpy(), sparse=[s.cpu().numpy() for s in sp]))
    # Sequence 0 is full: one more append reports a bad length and leaves it as it
    # was, while sequence 1 still grows.
    k_new, v_new = _new_rows(gen, 2, n_new), _new_rows(gen, 2, n_new)
    hs2.kv_append(k_new.to(dev), v_new.to(dev), cache, ws)
    assert hs2.STATUS[hs2.check_device_status(ws)] == "HS2_ERR_BAD_LENGTH"
    want = oracle.kv_append(dict(bits, lens=bits["lens"][1:], k=bits["k"][1:], v=bits["v"][1:],
                                 k_scale=None if bits["k_scale"] is None else bits["k_scale"][1:],
                                 v_scale=None if bits["v_scale"] is None else bits["v_scale"][1:]),
                            _bits_of(k_new)[1:], _bits_of(v_new)[1:])
    for key in ("lens", "k", "v", "k_scale", "v_scale"):
        if want[key] is not None:
            want[key] = np.concatenate([bits[key][:1], want[key]])
    _assert_cache_equal(cache, want)


# Block-level selection (the first-generation comparator): the GPU's block sets
# against the oracle's, and the sparse layers on the GPU's sets.
BLOCK_CASES = [
    dict(id="b1-L4096-h16-bf16", batch=1, max_len=4096, n_q=1, h_q=16, kv="bf16", seed=201,
         n_needles=8, needle_layout="uniform"),
    dict(id="ragged-b3-bf16", batch=3, max_len=5000, n_q=1, h_q=16, kv="bf16", seed=202,
         lens=[5000, 1217, 1153]),
    dict(id="h64-fp8-ragged", batch=2, max_len=3000, n_q=1, h_q=64, kv="fp8", seed=203,
         lens=[3000, 2901]),
    dict(id="h32-append4", batch=1, max_len=2500, n_q=4, h_q=32, kv="bf16", seed=204),
    dict(id="append13-h16-ragged", batch=2, max_len=7000, n_q=13, h_q=16, kv="bf16", seed=205,
         lens=[7000, 2222]),
    dict(id="h48-fp8", batch=2, max_len=1800, n_q=2, h_q=48, kv="fp8", seed=206,
         lens=[1800, 1500]),
    dict(id="h128-bf16", batch=1, max_len=2000, n_q=1, h_q=128, kv="bf16", seed=207),
    dict(id="tiny-window4-k8-block4", batch=2, max_len=48, n_q=3, h_q=16, kv="bf16", seed=208,
         lens=[48, 13], window=4, k_sel=8, block=4),
    dict(id="block16-fp8", batch=1, max_len=6000, n_q=1, h_q=16, kv="fp8", seed=209, block=16),
    dict(id="short-contexts", batch=4, max_len=1300, n_q=1, h_q=16, kv="bf16", seed=210,
         lens=[1, 1152, 1153, 1217]),
]


def run_gpu_blocks(inp: workloads.Inputs, block: int):
    dev = torch.device("cuda:0")
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev),
                      None if inp.k_scale is None else inp.k_scale.to(dev),
                      None if inp.v_scale is None else inp.v_scale.to(dev))
    ws = hs2.alloc_workspace(cache, inp.n_q, inp.h_q, inp.window, inp.k_sel)
    out, idx, lse = hs2.full_attn_select_blocks(inp.q.to(dev), cache, inp.window, inp.k_sel,
                                                block, inp.sm_scale, ws)
    sp = [hs2.sparse_attn(ql.to(dev), cache, idx, ws, inp.sm_scale) for ql in inp.q_layers]
    status = hs2.check_device_status(ws)
    return dict(out=out.cpu().numpy(), idx=idx.cpu().numpy(), lse=lse.cpu().numpy(),
                sparse=[x.cpu().numpy() for x in sp]), status


def compare_blocks(inp: workloads.Inputs, res: dict, block: int):
    bits = workloads.numpy_bits(inp)
    ref = oracle.full_attn_select(bits, keep_importance=True, block=block)
    tol = TOL[inp.kv]
    assert np.abs(res["out"] - ref["out"]).max() < tol
    assert np.abs(res["lse"] - ref["lse"]).max() < LSE_TOL
    n_exact = 0
    for b in range(inp.batch):
        L = int(inp.lens[b])
        for i in range(inp.n_q):
            p = L - inp.n_q + i
            msg = check_block_index_set(res["idx"][b, i], ref["idx"][b, i],
                                        ref["imp"][b * inp.n_q + i], p, inp.window, inp.k_sel,
                                        block)
            assert msg is None, f"(b={b}, i={i}, p={p}): {msg}"
            n_exact += int(np.array_equal(res["idx"][b, i], ref["idx"][b, i]))
    for li, ql in enumerate(bits["q_layers"]):
        want = oracle.sparse_attn(bits, ql, res["idx"])
        assert np.abs(res["sparse"][li] - want).max() < tol, f"sparse layer {li}"
    return n_exact


@pytest.mark.parametrize("case", BLOCK_CASES, ids=lambda c: c["id"])
def test_block_selection_matches_oracle(case):
    kw = {k: v for k, v in case.items() if k not in ("id", "block")}
    block = case.get("block", 64)
    inp = workloads.make_inputs(n_sparse=2, **kw)
    res, status = run_gpu_blocks(inp, block)
    assert status == 0
    compare_blocks(inp, res, block)


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_block_selection_zero_query_keeps_lowest_blocks(kv):
    inp = workloads.make_inputs(1, 3000, n_q=1, h_q=16, kv=kv, seed=211, q_zero=True)
    res, status = run_gpu_blocks(inp, 64)
    assert status == 0
    want = np.concatenate([np.arange(1024), np.arange(3000 - 128, 3000)])
    assert res["idx"][0, 0].tolist() == want.tolist()


@pytest.mark.parametrize("kv,h_q", [("bf16", 16), ("fp8", 64)])
def test_separate_full_layer_and_selection_match_oracle(kv, h_q):
    """hs2_full_attn then hs2_select (the two halves of hs2_full_attn_select) on one
    60000-key row: the full layer's CTAs share the row's tiles out at run time (the stored
    logits of the 16-head step are indexed by position, whoever computed them)."""
    dev = torch.device("cuda:0")
    inp = workloads.make_inputs(1, 60000, n_q=1, h_q=h_q, kv=kv, seed=213, n_sparse=1)
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev),
                      None if inp.k_scale is None else inp.k_scale.to(dev),
                      None if inp.v_scale is None else inp.v_scale.to(dev))
    ws = hs2.alloc_workspace(cache, 1, h_q)
    q = inp.q.to(dev)
    lse = torch.empty(1, 1, h_q, dtype=torch.float32, device=dev)
    out = hs2.full_attn(q, cache, 128, 1024, inp.sm_scale, ws, lse=lse)
    idx = hs2.select(q, cache, ws, 128, 1024, inp.sm_scale)
    sp = [hs2.sparse_attn(inp.q_layers[0].to(dev), cache, idx, ws, inp.sm_scale)]
    assert hs2.check_device_status(ws) == 0
    compare(inp, dict(out=out.cpu().numpy(), idx=idx.cpu().numpy(), lse=lse.cpu().numpy(),
                      sparse=[x.cpu().numpy() for x in sp]))


def test_block_then_token_selection_share_a_workspace():
    """Block mode leaves the selection state clean: a token-level call on the same
    workspace right after it still matches the oracle."""
    dev = torch.device("cuda:0")
    inp = workloads.make_inputs(2, 5000, n_q=1, h_q=16, kv="bf16", seed=212, n_sparse=1,
                                lens=[5000, 3000])
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev))
    ws = hs2.alloc_workspace(cache, 1, 16)
    q = inp.q.to(dev)
    hs2.full_attn_select_blocks(q, cache, 128, 1024, 64, inp.sm_scale, ws)
    out, idx, lse = hs2.full_attn_select(q, cache, 128, 1024, inp.sm_scale, ws)
    sp = [hs2.sparse_attn(inp.q_layers[0].to(dev), cache, idx, ws, inp.sm_scale)]
    assert hs2.check_device_status(ws) == 0
    compare(inp, dict(out=out.cpu().numpy(), idx=idx.cpu().numpy(), lse=lse.cpu().numpy(),
                      sparse=[x.cpu().numpy() for x in sp]))


# Chunked prefill of the full layer (no selection): many new tokens per sequence.
PREFILL_CASES = [
    dict(id="L4096-chunk512-h16", batch=1, max_len=4096, n_q=512, h_q=16, seed=301),
    dict(id="ragged-chunk300-h32", batch=2, max_len=3000, n_q=300, h_q=32, seed=302,
         lens=[3000, 1500]),
    dict(id="whole-context-1024-h64", batch=1, max_len=1024, n_q=1024, h_q=64, seed=303),
    dict(id="chunk37-h128", batch=1, max_len=1500, n_q=37, h_q=128, seed=304),
    dict(id="chunk129-h16-ragged", batch=2, max_len=2000, n_q=129, h_q=16, seed=305,
         lens=[2000, 129]),
    dict(id="single-token-h48", batch=3, max_len=700, n_q=1, h_q=48, seed=306,
         lens=[700, 1, 333]),
]


@pytest.mark.parametrize("case", PREFILL_CASES, ids=lambda c: c["id"])
def test_prefill_matches_oracle(case):
    kw = {k: v for k, v in case.items() if k != "id"}
    inp = workloads.make_inputs(kv="bf16", n_sparse=0, **kw)
    dev = torch.device("cuda:0")
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev))
    ws = hs2.prefill_workspace(cache, inp.n_q, inp.h_q)
    out, lse = hs2.prefill_attn(inp.q.to(dev), cache, inp.sm_scale, ws)
    assert hs2.check_device_status(ws) == 0
    ref = oracle.prefill_attn(workloads.numpy_bits(inp))
    assert np.abs(out.cpu().numpy() - ref["out"]).max() < TOL["bf16"]
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() < LSE_TOL


def test_prefill_reports_a_sequence_shorter_than_the_chunk():
    inp = workloads.make_inputs(2, 200, n_q=64, h_q=16, seed=307, n_sparse=0, lens=[200, 50])
    dev = torch.device("cuda:0")
    cache = hs2.Cache(inp.k.to(dev), inp.v.to(dev), inp.lens.to(dev))
    ws = hs2.prefill_workspace(cache, 64, 16)
    hs2.prefill_attn(inp.q.to(dev), cache, inp.sm_scale, ws)
    assert hs2.STATUS[hs2.check_device_status(ws)] == "HS2_ERR_BAD_LENGTH"
