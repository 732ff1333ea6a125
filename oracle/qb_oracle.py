"""CPU oracle of the Quantile Balancing bias update (test infrastructure only).

Sources (web pages; cited by title and section):

[K3-896] "Kimi K3の896エキスパートを「896人の専門家」と呼ぶと何がズレるか、
         ルーターは何を選んでいるのか" (lilting.ch), section
   "ルーター専用の独立訓練はない": for every expert, the boundary at which it
   receives its target number of tokens is found from quantiles of the router
   scores, and the selection bias is updated from it; the quantiles are
   computed during training only (the bias is frozen at inference).
[K3-2axis] "Kimi K3の二軸スケーリング戦略とは何か" (studioglobal.ai), section
   "Stable LatentMoE：条件付きの大容量を安定させる": quantile-based load
   balancing of the batch's expert assignment.
[K3-report] Kimi K3 tech-report summary (jiwasawa.github.io), section
   "幅のスケーリング：Stable LatentMoE", item "Quantile Balancing (QB)": no
   auxiliary loss; quantiles are computed directly from the histogram of the
   router's score margins and each expert's bias is adjusted.

Reading (the pages give no formula; each point is also listed in the design
notes):
  * Keys are the selection keys of the forward pass, fl32(s + b), with ties to
    the lower expert index.
  * The score margin of expert e for token t is m = key_e - theta, where theta
    is the k-th largest key among the OTHER experts of the token: the
    (k+1)-th largest key of the token if e is among its top k, else its k-th
    largest.  Token t selects e exactly when m > 0, and moving b_e alone by
    delta moves every margin of e by delta, so e then receives the tokens
    with m > -delta.
  * Target count per expert: c = floor(T * k / E) tokens (a balanced batch).
  * The boundary is the quantile of e's margins at rank c: q_e is taken
    between the c-th and (c+1)-th largest margin, and the update is
    b_e <- b_e - q_e (applied to every expert at once).
  * The quantile is read from a histogram of the margins (nb equal bins on
    [lo, hi), margins outside clamped to the end bins) with the margins
    spread evenly inside a bin: if A margins lie in the bins above bin j and
    bin j (lower edge lo + j*w) holds n_j of them with A < c <= A + n_j,
    then q = lo + w * (j + 1 - (c - A) / n_j).  The exact quantile (the
    midpoint of the c-th and (c+1)-th largest margin) is given too; when the
    c-th margin lies inside [lo, hi) the two differ by at most one bin width
    plus half the gap between the c-th and (c+1)-th margins (q lies in the
    c-th margin's bin).
  * Binning decides an integer from floating point, so it is written as the
    device evaluates it, in fp32: bin = clamp(floor(fl32(fl32(m - lo) * inv_w)),
    0, nb - 1) with m = fl32(key_e - theta) and inv_w = fl32(nb / (hi - lo)).
"""
from __future__ import annotations

import numpy as np

__all__ = ["qb_keys", "qb_margins", "qb_target", "qb_quantile_exact", "qb_rank_margins", "qb_inv_width", "qb_histogram",
           "qb_quantile_from_hist", "qb_bias_update"]


def qb_keys(s32, b32) -> np.ndarray:
    """Selection keys fl32(s + b) [T, E]; a NaN key ranks below every number."""
    s32 = np.asarray(s32, dtype=np.float32)
    b32 = np.asarray(b32, dtype=np.float32)
    key = (s32 + b32[None, :]).astype(np.float32)
    key[np.isnan(key)] = -np.inf
    return key


def qb_margins(s32, b32, k: int):
    """Score margins of every (token, expert).

    Returns (m32 [T,E] float32 = fl32(key - theta), m64 [T,E] float64 = the
    exact difference, selected [T,E] bool = e among the token's top k)."""
    key = qb_keys(s32, b32)
    T, E = key.shape
    if not 0 < k < E:
        raise ValueError("the margin needs 0 < k < E")
    # descending by key, ties to the lower index: sort by (-key, index)
    order = np.lexsort((np.broadcast_to(np.arange(E), (T, E)), -key.astype(np.float64)), axis=1)
    kth = key[np.arange(T), order[:, k - 1]]
    k1th = key[np.arange(T), order[:, k]]
    selected = np.zeros((T, E), dtype=bool)
    np.put_along_axis(selected, order[:, :k], True, axis=1)
    theta = np.where(selected, k1th[:, None], kth[:, None]).astype(np.float32)
    m64 = key.astype(np.float64) - theta.astype(np.float64)
    with np.errstate(invalid="ignore"):
        m32 = (key - theta).astype(np.float32)
    return m32, m64, selected


def qb_target(T: int, k: int, E: int) -> int:
    """Balanced tokens per expert, c = floor(T k / E)."""
    return (T * k) // E


def qb_quantile_exact(m64: np.ndarray, c: int) -> np.ndarray:
    """Per expert, the midpoint of its c-th and (c+1)-th largest margin."""
    lo_hi = qb_rank_margins(m64, c)
    return 0.5 * (lo_hi[0] + lo_hi[1])


def qb_rank_margins(m64: np.ndarray, c: int):
    """Per expert, (c-th largest margin, (c+1)-th largest margin)."""
    srt = -np.sort(-m64, axis=0)  # descending per column
    if not 1 <= c < srt.shape[0]:
        raise ValueError("target count must be in [1, T)")
    return srt[c - 1], srt[c]


def qb_inv_width(nb: int, lo: float, hi: float) -> np.float32:
    return np.float32(nb / (hi - lo))


def qb_histogram(m32: np.ndarray, nb: int, lo: float, hi: float) -> np.ndarray:
    """Counts [E, nb] of the margins of each expert (fp32 binning, clamped)."""
    inv_w = qb_inv_width(nb, lo, hi)
    with np.errstate(invalid="ignore", over="ignore"):
        u = ((m32 - np.float32(lo)).astype(np.float32) * inv_w).astype(np.float32)
        u = np.nan_to_num(u, nan=0.0, posinf=float(nb), neginf=-1.0)
    b = np.clip(np.floor(u), 0, nb - 1).astype(np.int64)  # [T, E]
    T, E = m32.shape
    counts = np.zeros((E, nb), dtype=np.int64)
    np.add.at(counts, (np.broadcast_to(np.arange(E), (T, E)), b), 1)
    return counts


def qb_quantile_from_hist(counts: np.ndarray, c: int, lo: float, hi: float) -> np.ndarray:
    """Per expert, the rank-c boundary read from its histogram (fp64)."""
    E, nb = counts.shape
    w = (hi - lo) / nb
    q = np.empty(E, dtype=np.float64)
    for e in range(E):
        above = 0
        for j in range(nb - 1, -1, -1):
            n = int(counts[e, j])
            if above + n >= c:
                q[e] = lo + w * ((j + 1) - (c - above) / n)
                break
            above += n
        else:
            raise ValueError("fewer margins than the target count")
    return q


def qb_bias_update(s32, b32, k: int, nb: int, lo: float, hi: float) -> dict:
    """One Quantile Balancing step on a batch of router scores."""
    m32, m64, selected = qb_margins(s32, b32, k)
    T, E = m32.shape
    c = qb_target(T, k, E)
    counts = qb_histogram(m32, nb, lo, hi)
    q = qb_quantile_from_hist(counts, c, lo, hi)
    return {"counts": counts, "q": q, "bias": np.asarray(b32, dtype=np.float64) - q, "target": c,
            "q_exact": qb_quantile_exact(m64, c), "rank_gap": np.subtract(*qb_rank_margins(m64, c)),
            "selected": selected, "m64": m64}
