"""Column-interval masks for attn_fwd_colmask: builders and visible-pair counts.

A mask is an int32 array [B, Hm, Nk, 4]; entry (b, h, j) = (lo1, hi1, lo2, hi2)
hides key j from the query rows lo1 <= i < hi1 and lo2 <= i < hi2 (an interval
with lo >= hi is empty).  The kernel's causal flag additionally hides keys
j > i.  This module only builds such arrays and counts the pairs they leave
visible (for FLOP accounting); it holds no attention arithmetic.
"""
from __future__ import annotations

import numpy as np

ROW_MAX = np.iinfo(np.int32).max  # an interval end past every query row


def empty(B: int, Hm: int, Nk: int) -> np.ndarray:
    """No key hidden from any row."""
    return np.zeros((B, Hm, Nk, 4), dtype=np.int32)


def documents(lengths_per_batch, Nk: int, bidirectional: bool = False) -> np.ndarray:
    """Document mask [B, 1, Nk, 4]: the sequence is cut into documents of the
    given lengths (per batch entry; they must sum to Nk) and no row sees a key
    of another document.  With the kernel's causal flag this is the usual
    block-diagonal causal mask; bidirectional=True also hides each key from the
    rows before its document (so it works without the causal flag)."""
    out = empty(len(lengths_per_batch), 1, Nk)
    for b, lens in enumerate(lengths_per_batch):
        assert sum(lens) == Nk, "document lengths must cover the sequence"
        start = 0
        for n in lens:
            out[b, 0, start:start + n, 0] = start + n
            out[b, 0, start:start + n, 1] = ROW_MAX
            if bidirectional:
                out[b, 0, start:start + n, 2] = 0
                out[b, 0, start:start + n, 3] = start
            start += n
    return out


def document_lengths(seed: int, n: int, lo: int, hi: int) -> list:
    """Document lengths uniform in [lo, hi] from the counter-based generator
    (draw t of tensor id "len"), the last one cut so that they sum to n."""
    from . import inputs
    out, t = [], 0
    while sum(out) < n:
        u = inputs.uniform_at(seed, "len", np.array([t], dtype=np.int64))[0]
        out.append(min(int(lo + (hi - lo) * u), n - sum(out)))
        t += 1
    return out


def prefix_lm(B: int, Nk: int, prefix: int) -> np.ndarray:
    """Prefix-LM (use without the causal flag): every row sees the first
    `prefix` keys; a key j >= prefix is seen only by rows i >= j."""
    out = empty(B, 1, Nk)
    j = np.arange(prefix, Nk, dtype=np.int32)
    out[:, 0, prefix:, 1] = j  # rows [0, j)
    return out


def band(B: int, Nk: int, window_left: int, window_right: int) -> np.ndarray:
    """The key band i - window_left <= j <= i + window_right (-1: no bound) as
    column intervals: key j is hidden from rows i > j + window_left and from
    rows i < j - window_right."""
    out = empty(B, 1, Nk)
    j = np.arange(Nk, dtype=np.int64)
    if window_left >= 0:
        out[:, 0, :, 0] = np.minimum(j + window_left + 1, ROW_MAX)
        out[:, 0, :, 1] = ROW_MAX
    if window_right >= 0:
        out[:, 0, :, 2] = 0
        out[:, 0, :, 3] = np.maximum(j - window_right, 0)
    return out


def random_intervals(seed: int, B: int, Hm: int, Nq: int, Nk: int) -> np.ndarray:
    """Seeded stress mask: per key, two intervals with random ends in
    [-Nq/8, 9Nq/8) (some empty, some covering all rows), drawn from the
    counter-based generator."""
    from . import inputs
    n = B * Hm * Nk * 4
    u = inputs.uniform_at(seed, "mask", np.arange(n, dtype=np.int64)).reshape(B, Hm, Nk, 4)
    ends = np.floor((u * 1.25 - 0.125) * Nq).astype(np.int64)
    lo = np.minimum(ends[..., 0::2], ends[..., 1::2])
    hi = np.maximum(ends[..., 0::2], ends[..., 1::2])
    out = np.empty((B, Hm, Nk, 4), dtype=np.int32)
    out[..., 0], out[..., 1] = lo[..., 0], hi[..., 0]
    out[..., 2], out[..., 3] = lo[..., 1], hi[..., 1]
    return out


def visible_per_key(cols: np.ndarray, Nq: int, causal: bool) -> np.ndarray:
    """Rows 0..Nq-1 that see each key: cols [..., Nk, 4] -> int64 [..., Nk].
    Counts Nq minus the union of the key's two intervals (and, when causal, the
    rows i < j), each clipped to [0, Nq)."""
    cols = np.asarray(cols, dtype=np.int64)
    nk = cols.shape[-2]
    j = np.broadcast_to(np.arange(nk, dtype=np.int64), cols.shape[:-1])
    starts = [cols[..., 0], cols[..., 2], np.zeros_like(j)]
    ends = [cols[..., 1], cols[..., 3], j if causal else np.zeros_like(j)]
    s = np.stack([np.clip(x, 0, Nq) for x in starts], axis=-1)
    e = np.stack([np.clip(x, 0, Nq) for x in ends], axis=-1)
    e = np.maximum(e, s)  # empty intervals -> zero length
    order = np.argsort(s, axis=-1)
    s = np.take_along_axis(s, order, axis=-1)
    e = np.take_along_axis(e, order, axis=-1)
    hidden = np.zeros(cols.shape[:-1], dtype=np.int64)
    reach = np.zeros(cols.shape[:-1], dtype=np.int64)  # end of the union so far
    for t in range(3):
        lo = np.maximum(s[..., t], reach)
        hidden += np.maximum(e[..., t] - lo, 0)
        reach = np.maximum(reach, e[..., t])
    return Nq - hidden


def visible_per_row(cols: np.ndarray, rows, causal: bool) -> np.ndarray:
    """Keys seen by each of the given query rows: cols [Nk, 4] -> int64 [n]."""
    cols = np.asarray(cols, dtype=np.int64)
    i = np.asarray(rows, dtype=np.int64)[:, None]
    j = np.arange(cols.shape[0], dtype=np.int64)[None, :]
    hidden = ((cols[None, :, 0] <= i) & (i < cols[None, :, 1])) | \
             ((cols[None, :, 2] <= i) & (i < cols[None, :, 3]))
    if causal:
        hidden |= j > i
    return cols.shape[0] - hidden.sum(axis=1)


def visible_pairs(cols: np.ndarray, Nq: int, causal: bool) -> np.ndarray:
    """Visible (query, key) pairs per mask row: [B, Hm, Nk, 4] -> [B, Hm]."""
    return visible_per_key(cols, Nq, causal).sum(axis=-1)
