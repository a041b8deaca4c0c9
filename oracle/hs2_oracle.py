"""Float64 CPU oracle for the HySparse2 hybrid-block decode step.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline legs of ``bench.py`` may import this module.  The CUDA path neither
imports it nor shares any code, table or helper with it; the product fails
loudly when its CUDA library is missing instead of falling back to this.

It is a plain, slow, obviously correct restatement in numpy float64 of what the
step computes.  Inputs arrive as raw storage (bf16 as uint16 bit patterns, FP8
as uint8 E4M3 codes) and are widened exactly to float64 before any arithmetic.

Sources, cited below by tag (web pages about the HySparse2 architecture paper):
  [SP]  "Luo Fuli Teases Xiaomi MiMo-V3 Architecture: HySparse2 Enables Early
        Prefill Exit" (ai.synthepulse.app, story 13379).
  [TNfr] toolnavs.com article 2080 (French), sections "Ce que fait HySparse2"
        and "Les chiffres mesurés".
  [TNko] toolnavs.com article 2080 (Korean), section "HySparse2가 한 일".
  [RAT] readaitime.com news of 2026-09-24 (Traditional Chinese), paragraphs on
        two-level KV sharing and on the forced recent window.

What the pages fix:
  * A Cross-Decoder hybrid block is one full-attention layer followed by several
    sparse-attention layers; the full layer picks important positions from its
    own attention scores and the sparse layers reuse its KV cache and its
    selected indices, with no trained selector ([TNfr] "Ce que fait HySparse2",
    KV Reuse paragraph; [TNko] same section; [SP] paragraph on KV Reuse).
  * Selection is per token, not per block; the most recent 128 tokens are always
    kept, plus 1024 tokens chosen outside that window ([TNfr] and [TNko], paragraph
    on selection granularity; [SP] paragraph on token granularity; [RAT]).
  * The full layer is MQA: one shared K/V head ([TNfr] "Les chiffres mesurés").
  * The KV cache may be FP8 ([SP] paragraph on cost at 1M tokens).

Readings where the pages are silent (each also listed in the design notes):
  * Importance of key j is max over query heads h of exp(s_hj - lse_h), the full
    layer's softmax probability; ties go to the lower position.
  * The 1024 are chosen among positions [0, p-128] (outside the window), so a
    full set has 1152 indices; with p+1 <= 1152 every position [0, p] is kept.
  * The window includes the current token: [max(0, p-127), p].
  * Index sets are ascending and padded with -1 to window + k_sel entries.
  * s_hj = sm_scale * q_h . k_j with sm_scale the float32 value passed in.
  * FP8 is OCP E4M3 ("fn"); a stored code times its per-token float32 scale is
    the key or value (the product is exact in float64).
  * Query token i of a sequence of length L (n_q query tokens) sits at position
    p = L - n_q + i and sees keys [0, p] (the context includes the new tokens).
  * Sparse layers take a plain softmax over the selected rows only; -1 slots are
    skipped.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_to_f64", "e4m3_to_f64", "widen_cache", "attend", "importance",
    "select_top", "index_set", "block_index_set", "full_attn_select", "prefill_attn", "sparse_attn", "hybrid_block_step",
    "f32_to_e4m3", "quantize_row_e4m3", "kv_append",
]


# ----------------------------------------------------------------------------
# Exact widening of the storage formats.
# ----------------------------------------------------------------------------
def bf16_to_f64(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float64.  A bf16 value is the upper half of the
    IEEE binary32 pattern with the lower 16 bits zero, so the widening is exact."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(codes) -> np.ndarray:
    """OCP FP8 E4M3 ("fn") codes -> float64, from the format's definition:
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 is
    subnormal (m/8 * 2^-6); no infinities; S.1111.111 is NaN; max 448."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def widen_cache(rows, kv: str, scale=None) -> np.ndarray:
    """K or V rows [n, d] in storage format -> float64 values.
    For FP8 each row is its codes times that token's float32 scale."""
    if kv == "bf16":
        return bf16_to_f64(rows)
    if kv == "fp8":
        return e4m3_to_f64(rows) * np.asarray(scale, dtype=np.float32).astype(np.float64)[:, None]
    raise ValueError(kv)


# ----------------------------------------------------------------------------
# The full-attention layer (MQA) and the importance of each key.
# ----------------------------------------------------------------------------
def attend(q, keys, vals, sm_scale: float):
    """Softmax attention of h query heads over n keys of one shared K/V head.

    q [h, d], keys [n, d], vals [n, d] (float64).  Returns
    out [h, d], lse [h] (natural log), P [h, n] (probabilities), s [h, n] (logits).
    The full layer scores every key it can see ([SP] paragraph on full attention
    giving complete attention scores; [TNfr] "Ce que fait HySparse2")."""
    s = float(sm_scale) * (q @ keys.T)
    m = s.max(axis=1)
    lse = m + np.log(np.exp(s - m[:, None]).sum(axis=1))
    P = np.exp(s - lse[:, None])
    return P @ vals, lse, P, s


def importance(s, lse) -> np.ndarray:
    """I_j = max_h exp(s_hj - lse_h): a key's largest softmax probability over the
    query heads.  The pages only say the selection comes from the full layer's
    attention scores; this is the reading taken."""
    return np.exp(s - lse[:, None]).max(axis=0)


def select_top(imp, k: int) -> np.ndarray:
    """Positions of the min(k, n) largest importances, ordered by (importance
    descending, position ascending): ties go to the lower position."""
    n = imp.shape[0]
    order = np.lexsort((np.arange(n), -imp))
    return order[:min(k, n)]


def index_set(p: int, imp_outside, window: int, k_sel: int) -> np.ndarray:
    """Token-level index set of query position p: the forced recent window
    [max(0, p-window+1), p] plus the top-k_sel keys of [0, p-window] by importance
    ([TNfr]/[TNko] paragraph on selection granularity; [RAT] forced window),
    ascending, padded with -1 to window + k_sel entries."""
    w_lo = max(0, p - window + 1)
    n_out = w_lo                                  # |[0, p-window]|
    assert imp_outside.shape[0] == n_out
    chosen = select_top(imp_outside, k_sel)
    sel = np.union1d(chosen, np.arange(w_lo, p + 1))
    out = np.full(window + k_sel, -1, dtype=np.int64)
    out[:sel.shape[0]] = np.sort(sel)
    return out


def block_index_set(p: int, imp_outside, window: int, k_sel: int, block: int = 64) -> np.ndarray:
    """Block-level index set of query position p: the first-generation scheme that the
    pages set token-level selection against ([SP] paragraph on block selection, where a
    64-token block spends selection budget as a whole, and paragraph on the ablation at
    the same attention budget; [RAT] paragraph on Block vs Token selection).
    Positions [0, p-window] form aligned blocks [c*block, (c+1)*block), the last one cut
    at p-window.  A block's score is the largest importance among its positions (the
    pages do not say how a block is scored; this is the reading taken).  The
    k_sel // block best blocks, ties to the lower block, are kept whole, plus the
    forced window; ascending, padded with -1 to window + k_sel entries."""
    w_lo = max(0, p - window + 1)
    n_out = w_lo
    assert imp_outside.shape[0] == n_out
    n_blk = -(-n_out // block)
    scores = np.array([imp_outside[c * block:(c + 1) * block].max() for c in range(n_blk)])
    chosen = select_top(scores, k_sel // block) if n_blk else np.zeros(0, dtype=np.int64)
    parts = [np.arange(c * block, min((c + 1) * block, n_out)) for c in chosen]
    sel = np.union1d(np.concatenate(parts + [np.arange(w_lo, p + 1)]), [])
    out = np.full(window + k_sel, -1, dtype=np.int64)
    out[:sel.shape[0]] = np.sort(sel).astype(np.int64)
    return out


def _rows(bits: dict, b: int, hi: int, which: str):
    scale = bits.get(which + "_scale")
    sc = None if scale is None else scale[b, :hi]
    return widen_cache(bits[which][b, :hi], bits["kv"], sc)


def full_attn_select(bits: dict, keep_importance: bool = False, block: int = 1):
    """The full-attention layer of the hybrid block plus its selection: token level
    (block = 1, the pages' scheme) or whole blocks of ``block`` positions (the
    first-generation comparator, block_index_set).

    ``bits``: q uint16 [B, n_q, h, d]; k, v uint16 or uint8 [B, max_len, d];
    k_scale, v_scale float32 [B, max_len] or None; lens [B]; sm_scale; window;
    k_sel; kv ("bf16" | "fp8").
    Returns dict(out [B,n_q,h,d], lse [B,n_q,h], idx int64 [B,n_q,window+k_sel],
    and when asked, imp: list of per-(b,i) importance arrays over [0, p-window])."""
    q_all = bf16_to_f64(bits["q"])
    B, n_q, h, d = q_all.shape
    W, K = int(bits["window"]), int(bits["k_sel"])
    out = np.zeros((B, n_q, h, d))
    lse = np.zeros((B, n_q, h))
    idx = np.full((B, n_q, W + K), -1, dtype=np.int64)
    imps = []
    for b in range(B):
        L = int(bits["lens"][b])
        keys = _rows(bits, b, L, "k")
        vals = _rows(bits, b, L, "v")
        for i in range(n_q):
            p = L - n_q + i
            o, l, P, s = attend(q_all[b, i], keys[:p + 1], vals[:p + 1], bits["sm_scale"])
            out[b, i], lse[b, i] = o, l
            w_lo = max(0, p - W + 1)
            imp = importance(s[:, :w_lo], l)
            idx[b, i] = (index_set(p, imp, W, K) if block == 1
                         else block_index_set(p, imp, W, K, block))
            if keep_importance:
                imps.append(imp)
    res = dict(out=out, lse=lse, idx=idx)
    if keep_importance:
        res["imp"] = imps
    return res


def prefill_attn(bits: dict):
    """The full-attention layer over a chunk of n_q new tokens (chunked prefill of the
    Cross-Decoder's full layer): the same attention as full_attn_select -- token i at
    p = L - n_q + i sees keys [0, p] ([TNfr] "Ce que fait HySparse2": the full layer
    attends over the whole context) -- without the selection.  Returns dict(out
    [B, n_q, h, d], lse [B, n_q, h])."""
    q_all = bf16_to_f64(bits["q"])
    B, n_q, h, d = q_all.shape
    out = np.zeros((B, n_q, h, d))
    lse = np.zeros((B, n_q, h))
    for b in range(B):
        L = int(bits["lens"][b])
        keys = _rows(bits, b, L, "k")
        vals = _rows(bits, b, L, "v")
        for i in range(n_q):
            p = L - n_q + i
            out[b, i], lse[b, i], _, _ = attend(q_all[b, i], keys[:p + 1], vals[:p + 1],
                                                bits["sm_scale"])
    return dict(out=out, lse=lse)


def sparse_attn(bits: dict, q_layer_bits, idx) -> np.ndarray:
    """One reusing sparse-attention layer: its own queries attend only to the rows
    named by the shared index set, read from the same KV cache ([TNfr] KV Reuse
    paragraph; [RAT] two-level sharing).  Softmax over the selected rows only;
    -1 slots are skipped.  Returns out [B, n_q, h, d]."""
    q_all = bf16_to_f64(q_layer_bits)
    B, n_q, h, d = q_all.shape
    out = np.zeros((B, n_q, h, d))
    for b in range(B):
        L = int(bits["lens"][b])
        keys = _rows(bits, b, L, "k")
        vals = _rows(bits, b, L, "v")
        for i in range(n_q):
            sel = np.asarray(idx[b, i])
            sel = sel[sel >= 0]
            o, _, _, _ = attend(q_all[b, i], keys[sel], vals[sel], bits["sm_scale"])
            out[b, i] = o
    return out


# ----------------------------------------------------------------------------
# Appending new tokens to the cache (the step before the full layer in a decode
# loop), with FP8 quantisation of each new row.
# ----------------------------------------------------------------------------
def f32_to_e4m3(y) -> np.ndarray:
    """float32 values -> OCP E4M3 ("fn") codes, round to nearest with ties to the even
    code, magnitudes beyond the largest finite value (448) saturating to it.  From the
    format's definition: a magnitude below 2^-6 is a subnormal with quantum 2^-9; in
    [2^e, 2^(e+1)), -6 <= e <= 8, the quantum is 2^(e-3).  A magnitude that rounds up to
    the next power of two moves to the next exponent (its code is the next one)."""
    y = np.asarray(y, dtype=np.float32).astype(np.float64)
    sign = (y < 0) | ((y == 0) & np.signbit(y))
    a = np.abs(y)
    # exponent of the binade holding a (frexp: a = f 2^x, f in [0.5, 1)), clamped to the
    # subnormal range below 2^-6 and to the top binade
    e = (np.frexp(np.where(a > 0, a, 1.0))[1] - 1).astype(np.float64)
    e = np.clip(e, -6, 8)
    q = np.exp2(e - 3.0)                      # quantum of that binade (2^-9 below 2^-6)
    n = a / q                                 # exact: q is a power of two
    r = np.floor(n)
    frac = n - r
    r = np.where((frac > 0.5) | ((frac == 0.5) & (np.fmod(r, 2.0) == 1.0)), r + 1.0, r)
    mag = r * q                               # the rounded magnitude
    mag = np.minimum(mag, 448.0)              # saturate
    # encode the rounded magnitude: subnormal (exp field 0) or normal
    sub = mag < 2.0 ** -6
    code_sub = np.round(mag / 2.0 ** -9).astype(np.int64)       # 0..7 (8 would be normal)
    en = (np.frexp(np.where(mag > 0, mag, 1.0))[1] - 1).astype(np.float64)
    m = np.round((mag / np.exp2(en) - 1.0) * 8.0).astype(np.int64)
    code_norm = ((en.astype(np.int64) + 7) << 3) | m
    out = np.where(sub, code_sub, code_norm)
    out = np.where(sign, out | 0x80, out)
    return out.astype(np.uint8)


def quantize_row_e4m3(row_bits):
    """One new K or V row (bf16 bit patterns, [d]) -> (E4M3 codes [d], float32 scale)
    by per-token absolute-maximum scaling: s = amax / 448 and code = E4M3(x / s), both
    divisions in IEEE float32 (round to nearest even); an all-zero row gets s = 1.
    (The pages say only that the cache may be FP8; per-token amax scaling is this
    build's reading.)"""
    x = bf16_to_f64(row_bits).astype(np.float32)
    amax = np.float32(np.max(np.abs(x)))
    s = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(448.0))
    y = (x / s).astype(np.float32)
    return f32_to_e4m3(y), s


def kv_append(bits: dict, k_new_bits, v_new_bits) -> dict:
    """Appends n_new tokens per sequence: token i of sequence b goes to row
    lens[b] + i of K and V (FP8 caches store codes and per-token scales from
    quantize_row_e4m3), and lens[b] grows by n_new.  Returns the new cache dict
    (inputs unchanged)."""
    out = dict(bits)
    k_new = np.asarray(k_new_bits, dtype=np.uint16)
    v_new = np.asarray(v_new_bits, dtype=np.uint16)
    B, n_new, d = k_new.shape
    lens = np.asarray(bits["lens"]).astype(np.int64).copy()
    k = np.array(bits["k"], copy=True)
    v = np.array(bits["v"], copy=True)
    fp8 = bits["kv"] == "fp8"
    ks = np.array(bits["k_scale"], copy=True) if fp8 else None
    vs = np.array(bits["v_scale"], copy=True) if fp8 else None
    for b in range(B):
        for i in range(n_new):
            r = int(lens[b]) + i
            if fp8:
                k[b, r], ks[b, r] = quantize_row_e4m3(k_new[b, i])
                v[b, r], vs[b, r] = quantize_row_e4m3(v_new[b, i])
            else:
                k[b, r] = k_new[b, i]
                v[b, r] = v_new[b, i]
        lens[b] += n_new
    out.update(k=k, v=v, lens=lens.astype(np.asarray(bits["lens"]).dtype))
    if fp8:
        out.update(k_scale=ks, v_scale=vs)
    return out


def hybrid_block_step(bits: dict, block: int = 1):
    """One decode step of the hybrid block: full layer + selection (token level, or
    whole blocks of ``block`` positions), then every reusing sparse layer in order.
    Returns (full-layer dict, [sparse outputs])."""
    full = full_attn_select(bits, block=block)
    sparse = [sparse_attn(bits, ql, full["idx"]) for ql in bits["q_layers"]]
    return full, sparse
