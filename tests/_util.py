"""Shared helpers of the test-suite (no method arithmetic beyond comparisons)."""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_cases(name: str):
    """Parse a golden text fixture made of ``case ... end`` blocks."""
    cases, cur = [], None
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            line = raw.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            if key == "case":
                cur = {"name": vals[0]}
            elif key == "end":
                cases.append(cur)
                cur = None
            else:
                cur[key] = [float(v) if "." in v else int(v) for v in vals]
    return cases


def bf16_bits(x) -> np.ndarray:
    """float values that are exactly representable in bf16 -> uint16 bit patterns."""
    f = np.asarray(x, dtype=np.float32)
    b = f.view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (b >> 16).astype(np.uint16)


def check_index_set(gpu_idx, ora_idx, imp, p: int, window: int, k_sel: int,
                    rel_band: float = 1e-6):
    """Compare one index set with the oracle's under the tie band.

    ``imp`` are the oracle's float64 importances over [0, p-window].  If the gap
    between its k-th and (k+1)-th importance is at least ``rel_band`` relative,
    the sets must be equal.  Otherwise every key clearly above the k-th value
    must be present, every key clearly below absent, and the size exact.
    Returns None on success, else a message."""
    g = np.asarray(gpu_idx, dtype=np.int64)
    o = np.asarray(ora_idx, dtype=np.int64)
    nvalid = min(p + 1, window + k_sel)
    if not np.all(g[:nvalid] >= 0) or not np.all(g[nvalid:] == -1):
        return f"bad padding: {g[max(0, nvalid - 3):nvalid + 3]} (expected {nvalid} valid)"
    gv = g[:nvalid]
    if np.any(np.diff(gv) <= 0):
        return "indices not strictly ascending"
    if np.array_equal(g, o):
        return None
    w_lo = max(0, p - window + 1)
    if not np.all(np.isin(np.arange(w_lo, p + 1), gv)):
        return "forced window missing"
    n_c = w_lo
    kk = min(k_sel, n_c)
    if kk == n_c:
        return f"all outside keys should be kept; differs at {np.setxor1d(g, o)[:8]}"
    srt = np.sort(imp)[::-1]
    ik, ik1 = srt[kk - 1], srt[kk]
    if (ik - ik1) >= rel_band * ik:
        diff = np.setxor1d(gv, o[o >= 0])
        return f"index sets differ outside the tie band at {diff[:8]} (gap {(ik - ik1) / ik:.3e})"
    chosen = gv[gv < w_lo]
    if chosen.shape[0] != kk:
        return f"wrong number of selected keys {chosen.shape[0]} != {kk}"
    above = np.nonzero(imp > ik * (1 + rel_band))[0]
    below = np.nonzero(imp < ik * (1 - rel_band))[0]
    if not np.all(np.isin(above, chosen)):
        return "a key clearly above the k-th importance is missing"
    if np.any(np.isin(below, chosen)):
        return "a key clearly below the k-th importance is present"
    return None


def check_block_index_set(gpu_idx, ora_idx, imp, p: int, window: int, k_sel: int, block: int,
                          rel_band: float = 1e-6):
    """Compare one block-level index set with the oracle's under the tie band on
    block scores (a block's score: the largest of the oracle's float64 importances
    among its positions).  If the kb-th and (kb+1)-th block scores differ by at least
    ``rel_band`` relative (kb = k_sel // block) the sets must be equal; otherwise
    the GPU set must hold kb whole blocks, every block clearly above the kb-th score
    and none clearly below.  Returns None on success, else a message."""
    g = np.asarray(gpu_idx, dtype=np.int64)
    o = np.asarray(ora_idx, dtype=np.int64)
    gv = g[g >= 0]
    if np.any(np.diff(gv) <= 0):
        return "indices not strictly ascending"
    if not np.all(g[gv.size:] == -1):
        return "padding not at the end"
    if np.array_equal(g, o):
        return None
    w_lo = max(0, p - window + 1)
    if not np.all(np.isin(np.arange(w_lo, p + 1), gv)):
        return "forced window missing"
    n_blk = -(-w_lo // block)
    kb = k_sel // block
    if n_blk <= kb:
        return "every position should be kept"
    score = np.array([imp[c * block:(c + 1) * block].max() for c in range(n_blk)])
    srt = np.sort(score)[::-1]
    sk, sk1 = srt[kb - 1], srt[kb]
    if sk - sk1 >= rel_band * sk:
        return f"block sets differ outside the tie band at {np.setxor1d(g, o)[:8]}"
    outside = gv[gv < w_lo]
    kept = np.unique(outside // block)
    if kept.size != kb:
        return f"{kept.size} blocks kept, expected {kb}"
    for c in kept:
        if not np.array_equal(outside[outside // block == c],
                              np.arange(c * block, min((c + 1) * block, w_lo))):
            return f"block {c} not whole"
    lo, hi = sk * (1 - rel_band), sk * (1 + rel_band)
    if np.any(score[np.setdiff1d(np.arange(n_blk), kept)] > hi):
        return "a block clearly above the boundary was dropped"
    if np.any(score[kept] < lo):
        return "a block clearly below the boundary was kept"
    return None
