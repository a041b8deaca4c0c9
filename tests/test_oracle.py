"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle against a library routine, a closed form, a
hand-derived fixture or brute force, so that a plausible slip in it (a dropped
term, a wrong sign or index, a swapped operand) fails at least one of them.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from long_context_token_b200 import workloads
from _util import bf16_bits, read_cases

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- formats
def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan) and nan.sum() == 2
    assert np.array_equal(ours[~nan], ref[~nan])


def test_e4m3_decode_spec_points():
    # OCP E4M3: 0x7E is the largest finite value 448, 0x01 the smallest
    # subnormal 2^-9, 0x08 the smallest normal 2^-6, 0x38 is 1.0.
    v = oracle.e4m3_to_f64(np.array([0x7E, 0x01, 0x08, 0x38, 0xB8, 0x00, 0x80], np.uint8))
    assert list(v[:5]) == [448.0, 2.0 ** -9, 2.0 ** -6, 1.0, -1.0]
    assert v[5] == 0.0 and v[6] == 0.0


def test_bf16_widening_matches_torch():
    x = torch.randn(4096, generator=torch.Generator().manual_seed(1)) * 7
    b = x.to(torch.bfloat16)
    ours = oracle.bf16_to_f64(b.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(ours, b.to(torch.float64).numpy())


# ------------------------------------------------------ full attention
def _sdpa(q, k, v, scale, mask=None):
    """torch's scaled_dot_product_attention in float64: q [h, d], k/v [n, d]."""
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None],
        attn_mask=None if mask is None else torch.from_numpy(mask)[None], scale=scale)
    return out[0].numpy()


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_full_attention_matches_library_sdpa_with_causal_queries(kv):
    inp = workloads.make_inputs(2, 300, n_q=5, h_q=16, kv=kv, seed=3, lens=[300, 211])
    bits = workloads.numpy_bits(inp)
    res = oracle.full_attn_select(bits)
    q = oracle.bf16_to_f64(bits["q"])
    for b in range(2):
        L = int(bits["lens"][b])
        k = oracle.widen_cache(bits["k"][b, :L], kv, None if kv == "bf16" else bits["k_scale"][b, :L])
        v = oracle.widen_cache(bits["v"][b, :L], kv, None if kv == "bf16" else bits["v_scale"][b, :L])
        for i in range(5):
            p = L - 5 + i
            mask = np.zeros((16, L), dtype=bool)
            mask[:, :p + 1] = True
            ref = _sdpa(q[b, i], k, v, bits["sm_scale"], mask)
            np.testing.assert_allclose(res["out"][b, i], ref, rtol=0, atol=1e-12)
            s = bits["sm_scale"] * q[b, i] @ k[:p + 1].T
            lse_ref = torch.logsumexp(torch.from_numpy(s), dim=1).numpy()
            np.testing.assert_allclose(res["lse"][b, i], lse_ref, rtol=0, atol=1e-12)


def test_prefill_matches_library_sdpa_with_one_causal_mask():
    """The chunk's tokens all at once: one float64 SDPA call over every (token, head)
    row with the causal mask [row, key] = key <= position of the row's token."""
    n_q, h = 40, 16
    inp = workloads.make_inputs(2, 200, n_q=n_q, h_q=h, seed=31, lens=[200, 97])
    bits = workloads.numpy_bits(inp)
    res = oracle.prefill_attn(bits)
    q = oracle.bf16_to_f64(bits["q"])
    for b in range(2):
        L = int(bits["lens"][b])
        k = oracle.bf16_to_f64(bits["k"][b, :L])
        v = oracle.bf16_to_f64(bits["v"][b, :L])
        pos = np.repeat(L - n_q + np.arange(n_q), h)           # row = token * h + head
        mask = np.arange(L)[None, :] <= pos[:, None]
        ref = _sdpa(q[b].reshape(n_q * h, 128), k, v, bits["sm_scale"], mask)
        np.testing.assert_allclose(res["out"][b].reshape(n_q * h, 128), ref, rtol=0, atol=1e-12)
        s = bits["sm_scale"] * q[b].reshape(n_q * h, 128) @ k.T
        s[~mask] = -np.inf
        lse_ref = torch.logsumexp(torch.from_numpy(s), dim=1).numpy()
        np.testing.assert_allclose(res["lse"][b].reshape(-1), lse_ref, rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(0)
    q, k, v = rng.standard_normal((8, 128)), rng.standard_normal((500, 128)), rng.standard_normal((500, 128))
    _, lse, P, _ = oracle.attend(q, k, v, 0.3)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(P > 0)


def test_zero_query_gives_mean_value_and_log_length():
    inp = workloads.make_inputs(1, 777, n_q=1, h_q=16, seed=5, q_zero=True)
    bits = workloads.numpy_bits(inp)
    res = oracle.full_attn_select(bits)
    v = oracle.bf16_to_f64(bits["v"][0])
    np.testing.assert_allclose(res["out"][0, 0], np.broadcast_to(v.mean(axis=0), (16, 128)), atol=1e-13)
    np.testing.assert_allclose(res["lse"][0, 0], math.log(777), atol=1e-13)


def test_identical_keys_give_uniform_attention():
    inp = workloads.make_inputs(1, 400, n_q=1, h_q=16, seed=6, identical_keys=True)
    bits = workloads.numpy_bits(inp)
    res = oracle.full_attn_select(bits)
    q = oracle.bf16_to_f64(bits["q"][0, 0])
    k0 = oracle.bf16_to_f64(bits["k"][0, 0])
    v = oracle.bf16_to_f64(bits["v"][0])
    np.testing.assert_allclose(res["out"][0, 0], np.broadcast_to(v.mean(axis=0), (16, 128)), atol=1e-13)
    np.testing.assert_allclose(res["lse"][0, 0], bits["sm_scale"] * q @ k0 + math.log(400), atol=1e-12)


# ------------------------------------------------------------ selection
def _bits_from_case(c):
    L, W, K = c["len"][0], c["window"][0], c["k_sel"][0]
    x, y = np.array(c["x"], float), np.array(c["y"], float)
    q = np.zeros((1, 1, 2, 128), np.float32)
    q[0, 0, 0, 0] = 2.0
    q[0, 0, 1, 1] = 2.0
    k = np.zeros((1, L, 128), np.float32)
    k[0, :, 0], k[0, :, 1] = x, y
    v = np.zeros((1, L, 128), np.float32)
    v[0, np.arange(L), np.arange(L)] = 1.0
    return dict(q=bf16_bits(q), k=bf16_bits(k), v=bf16_bits(v), k_scale=None, v_scale=None,
                lens=np.array([L]), sm_scale=0.5, window=W, k_sel=K, kv="bf16",
                q_layers=[])


@pytest.mark.parametrize("case", read_cases("selection_cases.txt"), ids=lambda c: c["name"])
def test_golden_selection_cases(case):
    bits = _bits_from_case(case)
    res = oracle.full_attn_select(bits)
    assert res["idx"][0, 0].tolist() == case["expected_idx"]
    # closed forms: y is a permutation of x, so both heads share lse = ln sum e^x,
    # and with one-hot values out_h[j] = exp(s_hj - lse).
    x, y = np.array(case["x"], float), np.array(case["y"], float)
    lse = math.log(np.exp(x).sum())
    np.testing.assert_allclose(res["lse"][0, 0], [lse, lse], atol=1e-14)
    L = case["len"][0]
    np.testing.assert_allclose(res["out"][0, 0, 0, :L], np.exp(x - lse), atol=1e-15)
    np.testing.assert_allclose(res["out"][0, 0, 1, :L], np.exp(y - lse), atol=1e-15)


def _brute_force_selection(q, k, sm_scale, p, W, K):
    """Selection of one query by definition, on tiny inputs: probabilities from
    torch.softmax (float64); key j is chosen iff fewer than K outside keys rank
    strictly before it in (importance desc, position asc)."""
    s = torch.from_numpy(sm_scale * q @ k[:p + 1].T)
    P = torch.softmax(s, dim=1).numpy()
    w_lo = max(0, p - W + 1)
    imp = [max(P[h, j] for h in range(P.shape[0])) for j in range(w_lo)]
    chosen = []
    for j in range(w_lo):
        rank = sum(1 for jj in range(w_lo) if imp[jj] > imp[j] or (imp[jj] == imp[j] and jj < j))
        if rank < K:
            chosen.append(j)
    return sorted(set(chosen) | set(range(w_lo, p + 1)))


@pytest.mark.parametrize("h", [1, 3, 16])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_selection_matches_brute_force_on_tiny_inputs(h, seed):
    W, K = 4, 8
    L = [48, 13, 9][seed]
    inp = workloads.make_inputs(1, 48, n_q=3, h_q=h, seed=20 + seed, lens=[L], window=W, k_sel=K)
    bits = workloads.numpy_bits(inp)
    res = oracle.full_attn_select(bits)
    q = oracle.bf16_to_f64(bits["q"][0])
    k = oracle.bf16_to_f64(bits["k"][0, :L])
    for i in range(3):
        p = L - 3 + i
        want = _brute_force_selection(q[i], k, bits["sm_scale"], p, W, K)
        got = res["idx"][0, i]
        assert got[got >= 0].tolist() == want
        assert np.all(got[len(want):] == -1)


def test_single_head_selection_is_argsort_of_logits():
    # With one head, lse is a common shift, so importance order = logit order.
    inp = workloads.make_inputs(1, 3000, n_q=1, h_q=1, seed=8, window=128, k_sel=1024)
    bits = workloads.numpy_bits(inp)
    res = oracle.full_attn_select(bits)
    q = oracle.bf16_to_f64(bits["q"][0, 0, 0])
    k = oracle.bf16_to_f64(bits["k"][0])
    s = k[:3000 - 128] @ q
    top = np.argsort(-s, kind="stable")[:1024]
    want = np.sort(np.concatenate([top, np.arange(3000 - 128, 3000)]))
    assert np.array_equal(res["idx"][0, 0], want)


def test_zero_query_ties_go_to_lowest_positions():
    inp = workloads.make_inputs(1, 5000, n_q=2, h_q=16, seed=9, q_zero=True)
    bits = workloads.numpy_bits(inp)
    res = oracle.full_attn_select(bits)
    for i in range(2):
        p = 5000 - 2 + i
        want = np.concatenate([np.arange(1024), np.arange(p - 127, p + 1)])
        assert np.array_equal(res["idx"][0, i], want)


def test_planted_needles_are_selected_and_window_present():
    w = workloads.WORKLOADS[1]
    inp = workloads.generate(w)
    bits = workloads.numpy_bits(inp)
    res = oracle.full_attn_select(bits)
    idx = res["idx"][0, 0]
    L = int(bits["lens"][0])
    assert len(inp.needles[0]) == 8
    for pos, _ in inp.needles[0]:
        assert pos in idx
    assert np.all(np.isin(np.arange(L - 128, L), idx))
    assert np.count_nonzero(idx >= 0) == 1152 and np.all(np.diff(idx) > 0)


@pytest.mark.parametrize("L", [1, 2, 127, 128, 129, 1151, 1152, 1153, 1300])
def test_index_set_size_window_and_order(L):
    inp = workloads.make_inputs(1, 1300, n_q=1, h_q=16, seed=10, lens=[L])
    bits = workloads.numpy_bits(inp)
    idx = oracle.full_attn_select(bits)["idx"][0, 0]
    p = L - 1
    nvalid = min(p + 1, 1152)
    assert np.all(idx[:nvalid] >= 0) and np.all(idx[nvalid:] == -1)
    assert np.all(np.diff(idx[:nvalid]) > 0) and idx[nvalid - 1] == p
    assert np.all(np.isin(np.arange(max(0, p - 127), p + 1), idx))


# ------------------------------------------------------------ sparse layers
@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_sparse_equals_full_when_budget_covers_context(kv):
    inp = workloads.make_inputs(2, 1152, n_q=2, h_q=16, kv=kv, n_sparse=1, seed=11, lens=[1152, 700])
    bits = workloads.numpy_bits(inp)
    full = oracle.full_attn_select(bits)
    # A sparse layer that reuses the full layer's own queries must reproduce it.
    out = oracle.sparse_attn(bits, bits["q"], full["idx"])
    np.testing.assert_allclose(out, full["out"], rtol=0, atol=1e-12)


def test_sparse_matches_library_sdpa_on_gathered_rows():
    inp = workloads.make_inputs(1, 6000, n_q=1, h_q=16, kv="fp8", n_sparse=1, seed=12)
    bits = workloads.numpy_bits(inp)
    full = oracle.full_attn_select(bits)
    out = oracle.sparse_attn(bits, bits["q_layers"][0], full["idx"])
    sel = full["idx"][0, 0]
    sel = sel[sel >= 0]
    k = oracle.e4m3_to_f64(bits["k"][0, sel]) * bits["k_scale"][0, sel].astype(np.float64)[:, None]
    v = oracle.e4m3_to_f64(bits["v"][0, sel]) * bits["v_scale"][0, sel].astype(np.float64)[:, None]
    ref = _sdpa(oracle.bf16_to_f64(bits["q_layers"][0][0, 0]), k, v, bits["sm_scale"])
    np.testing.assert_allclose(out[0, 0], ref, rtol=0, atol=1e-12)


# ------------------------------------------------------- block-level selection
@pytest.mark.parametrize("case", read_cases("block_selection_cases.txt"), ids=lambda c: c["name"])
def test_golden_block_selection_cases(case):
    bits = _bits_from_case(case)
    res = oracle.full_attn_select(bits, block=case["block"][0])
    assert res["idx"][0, 0].tolist() == case["expected_idx"]


@pytest.mark.parametrize("seed", range(6))
def test_block_size_one_is_token_selection(seed):
    rng = np.random.default_rng(seed)
    for p, W, K in ((300, 128, 64), (40, 4, 8), (9, 4, 8), (2000, 128, 1024)):
        n = max(0, p - W + 1)
        imp = rng.choice([0.1, 0.2, 0.3], size=n) * rng.integers(1, 4, size=n)  # many ties
        assert np.array_equal(oracle.block_index_set(p, imp, W, K, 1),
                              oracle.index_set(p, imp, W, K))


@pytest.mark.parametrize("seed", range(4))
def test_block_selection_keeps_whole_best_blocks(seed):
    """Invariants of the block set on random importances with ties: the kept outside
    positions are whole blocks (the cut last block counting whole), as many as the
    budget allows; no dropped block scores above a kept one, and among equal scores
    the kept blocks are the lower ones; the window is present; ascending; padded."""
    rng = np.random.default_rng(100 + seed)
    W, K, blk = 128, 1024, 64
    for p in (127, 128, 1151, 1152, 1300, 5000, 20000):
        w_lo = max(0, p - W + 1)
        imp = rng.integers(0, 50, size=w_lo) / 50.0
        got = oracle.block_index_set(p, imp, W, K, blk)
        valid = got[got >= 0]
        assert np.all(np.diff(valid) > 0) and np.all(got[valid.size:] == -1)
        assert np.all(np.isin(np.arange(w_lo, p + 1), valid))
        outside = valid[valid < w_lo]
        n_blk = -(-w_lo // blk)
        kept = np.unique(outside // blk)
        assert kept.size == min(n_blk, K // blk)
        for c in kept:
            assert np.array_equal(outside[outside // blk == c], np.arange(c * blk, min((c + 1) * blk, w_lo)))
        score = np.array([imp[c * blk:(c + 1) * blk].max() for c in range(n_blk)])
        dropped = np.setdiff1d(np.arange(n_blk), kept)
        if dropped.size and kept.size:
            assert score[kept].min() >= score[dropped].max()
            tie = score[kept].min()
            assert not np.any((score[dropped] == tie) & (dropped < kept[score[kept] == tie].max()))


def test_block_zero_query_keeps_lowest_blocks():
    inp = workloads.make_inputs(1, 3000, n_q=1, h_q=16, seed=7, q_zero=True)
    res = oracle.full_attn_select(workloads.numpy_bits(inp), block=64)
    p = 2999
    want = np.concatenate([np.arange(1024), np.arange(p - 127, p + 1)])
    assert res["idx"][0, 0].tolist() == want.tolist()


# -------------------------------------------- the pins catch planted mistakes
def _swap(monkeypatch, name, fn):
    monkeypatch.setattr(oracle.hs2_oracle, name, fn)


def test_pins_catch_min_over_heads(monkeypatch):
    _swap(monkeypatch, "importance", lambda s, lse: np.exp(s - lse[:, None]).min(axis=0))
    with pytest.raises(AssertionError):
        test_selection_matches_brute_force_on_tiny_inputs(3, 0)


def test_pins_catch_unnormalised_importance(monkeypatch):
    _swap(monkeypatch, "importance", lambda s, lse: np.exp(s).max(axis=0))
    with pytest.raises(AssertionError):
        test_selection_matches_brute_force_on_tiny_inputs(16, 0)


def test_pins_catch_reversed_tie_break(monkeypatch):
    def bad(imp, k):
        n = imp.shape[0]
        return np.lexsort((-np.arange(n), -imp))[:min(k, n)]
    _swap(monkeypatch, "select_top", bad)
    with pytest.raises(AssertionError):
        test_zero_query_ties_go_to_lowest_positions()


def test_pins_catch_window_off_by_one(monkeypatch):
    orig = oracle.hs2_oracle.index_set

    def bad(p, imp, window, k_sel):
        return orig(p, imp, window, k_sel) if p < window else np.concatenate(
            [orig(p, imp, window, k_sel)[1:], [-1]])
    _swap(monkeypatch, "index_set", bad)
    with pytest.raises(AssertionError):
        test_index_set_size_window_and_order(1300)


def test_pins_catch_dropped_scale(monkeypatch):
    orig = oracle.hs2_oracle.attend
    _swap(monkeypatch, "attend", lambda q, k, v, sc: orig(q, k, v, 1.0))
    with pytest.raises(AssertionError):
        test_full_attention_matches_library_sdpa_with_causal_queries("bf16")


def test_pins_catch_dropped_fp8_scale(monkeypatch):
    def bad(rows, kv, scale=None):
        return oracle.bf16_to_f64(rows) if kv == "bf16" else oracle.e4m3_to_f64(rows)
    _swap(monkeypatch, "widen_cache", bad)
    with pytest.raises(AssertionError):
        test_sparse_matches_library_sdpa_on_gathered_rows()


# ----------------------------------------------------------------------------
# Appending tokens: E4M3 encoding and per-token quantisation of the new rows.
# ----------------------------------------------------------------------------
def _to_bf16_bits(x) -> np.ndarray:
    """float32 array -> bf16 bit patterns (round to nearest even, through torch)."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _torch_e4m3(y):
    return torch.from_numpy(np.asarray(y, dtype=np.float32)).to(torch.float8_e4m3fn) \
        .view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_cast():
    """Round to nearest, ties to even, against torch's float8_e4m3fn cast (in range)."""
    rng = np.random.default_rng(7)
    mags = rng.choice(np.array([1e-5, 1e-3, 0.1, 1.0, 30.0, 300.0], dtype=np.float32), 100000)
    y = np.clip(rng.standard_normal(100000).astype(np.float32) * mags, -448, 448)
    assert np.array_equal(oracle.f32_to_e4m3(y), _torch_e4m3(y))


def test_e4m3_encode_inverts_decode_and_rounds_ties_to_even():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes).astype(np.float32)
    enc = oracle.f32_to_e4m3(vals)
    # every finite code decodes and re-encodes to itself (0x80 is -0)
    assert np.array_equal(enc, codes)
    # midpoints between neighbours of the same sign go to the even code
    pos = np.sort(oracle.e4m3_to_f64(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)
    got = oracle.f32_to_e4m3(mids)
    lo = np.arange(0, 0x7E, dtype=np.int64)
    want = np.where(lo % 2 == 0, lo, lo + 1)
    assert np.array_equal(got.astype(np.int64), want)
    assert np.array_equal(got, _torch_e4m3(mids))


def test_e4m3_encode_saturates_and_keeps_sign_of_zero():
    assert oracle.f32_to_e4m3(np.float32(500.0)) == 0x7E        # 448
    assert oracle.f32_to_e4m3(np.float32(-1e6)) == 0xFE
    assert oracle.f32_to_e4m3(np.float32(-1e-12)) == 0x80       # rounds to -0
    assert oracle.f32_to_e4m3(np.float32(2.0 ** -10)) == 0      # half of the smallest subnormal: even


def test_row_quantisation_scale_and_error_bound():
    rng = np.random.default_rng(3)
    x = rng.standard_normal(128).astype(np.float32) * 3
    bits = _to_bf16_bits(x)
    codes, s = oracle.quantize_row_e4m3(bits)
    xb = oracle.bf16_to_f64(bits)
    amax = np.abs(xb).max()
    assert np.float32(s) == np.float32(np.float32(amax) / np.float32(448.0))
    assert np.abs(oracle.e4m3_to_f64(codes)).max() == 448.0       # the amax maps to 448
    back = oracle.e4m3_to_f64(codes) * np.float64(s)
    # E4M3 keeps 3 mantissa bits: half-ulp error 2^-4 relative for normals, and an
    # absolute 2^-10 * s for subnormals
    err = np.abs(back - xb)
    assert np.all(err <= np.maximum(np.abs(xb) * 2.0 ** -4, 2.0 ** -10 * s) * (1 + 1e-9))
    zc, zs = oracle.quantize_row_e4m3(np.zeros(128, dtype=np.uint16))
    assert zs == np.float32(1.0) and not zc.any()


@pytest.mark.parametrize("kv", ["bf16", "fp8"])
def test_kv_append_writes_rows_and_grows_lengths(kv):
    inp = workloads.make_inputs(2, 600, n_q=1, h_q=16, kv=kv, seed=41, lens=[500, 321])
    bits = workloads.numpy_bits(inp)
    rng = np.random.default_rng(5)
    new = [_to_bf16_bits(rng.standard_normal((2, 3, 128))) for _ in range(2)]
    after = oracle.kv_append(bits, new[0], new[1])
    assert list(after["lens"]) == [503, 324]
    for b, L in enumerate([500, 321]):
        for i in range(3):
            for which, src in (("k", new[0]), ("v", new[1])):
                sc = after[which + "_scale"][b:b + 1, L + i] if kv == "fp8" else None
                got = oracle.widen_cache(after[which][b, L + i:L + i + 1], kv, sc)[0]
                want = oracle.bf16_to_f64(src[b, i])
                if kv == "bf16":
                    assert np.array_equal(got, want)
                else:
                    assert np.allclose(got, want, rtol=2 ** -4, atol=np.abs(want).max() * 2.0 ** -12)
        # rows before the old length are untouched
        assert np.array_equal(after["k"][b, :L], bits["k"][b, :L])
    assert np.array_equal(bits["lens"], [500, 321])                  # input unchanged


def test_pins_catch_truncating_encoder(monkeypatch):
    """A plausible mistake: rounding toward zero instead of to nearest-even."""
    def trunc(y):
        y = np.asarray(y, dtype=np.float32)
        t = torch.from_numpy(y).to(torch.float8_e4m3fn).float().numpy()
        over = np.abs(t) > np.abs(y)                   # rounded away from zero: step back
        codes = _torch_e4m3(y).astype(np.int64)
        codes = np.where(over & ((codes & 0x7F) > 0), codes - 1, codes)
        return codes.astype(np.uint8)
    monkeypatch.setattr(oracle, "f32_to_e4m3", trunc)
    with pytest.raises(AssertionError):
        test_e4m3_encode_inverts_decode_and_rounds_ties_to_even()


def test_pins_catch_block_mean_score(monkeypatch):
    def bad(p, imp_outside, window, k_sel, block=64):
        w_lo = max(0, p - window + 1)
        n_blk = -(-w_lo // block)
        scores = np.array([imp_outside[c * block:(c + 1) * block].mean() for c in range(n_blk)])
        chosen = oracle.select_top(scores, k_sel // block)
        parts = [np.arange(c * block, min((c + 1) * block, w_lo)) for c in chosen]
        sel = np.union1d(np.concatenate(parts + [np.arange(w_lo, p + 1)]), [])
        out = np.full(window + k_sel, -1, dtype=np.int64)
        out[:sel.shape[0]] = np.sort(sel).astype(np.int64)
        return out
    _swap(monkeypatch, "block_index_set", bad)
    case = read_cases("block_selection_cases.txt")[0]
    with pytest.raises(AssertionError):
        test_golden_block_selection_cases(case)
