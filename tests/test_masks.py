"""Column-interval mask builders and their visible-pair counts (CPU)."""
import numpy as np
import pytest

from exact_attention_152_b200 import masks


def dense_visible(cols, nq, causal):
    """Boolean [Nq, Nk] visibility of one mask row, element by element."""
    nk = cols.shape[0]
    vis = np.ones((nq, nk), dtype=bool)
    for j in range(nk):
        lo1, hi1, lo2, hi2 = (int(x) for x in cols[j])
        for i in range(nq):
            if lo1 <= i < hi1 or lo2 <= i < hi2 or (causal and j > i):
                vis[i, j] = False
    return vis


@pytest.mark.parametrize("causal", [False, True])
def test_visible_pairs_match_dense_count(causal):
    m = masks.random_intervals(3, 2, 3, 37, 29)
    got = masks.visible_pairs(m, 37, causal)
    for b in range(2):
        for h in range(3):
            assert got[b, h] == dense_visible(m[b, h], 37, causal).sum()


def test_visible_per_row_matches_dense():
    m = masks.random_intervals(4, 1, 1, 50, 33)[0, 0]
    rows = np.array([0, 3, 17, 49])
    for causal in (False, True):
        want = dense_visible(m, 50, causal)[rows].sum(axis=1)
        assert np.array_equal(masks.visible_per_row(m, rows, causal), want)


def test_random_intervals_cover_the_cases():
    m = masks.random_intervals(5, 1, 1, 64, 4096).reshape(-1, 4).astype(np.int64)
    assert np.all(m[:, 0] <= m[:, 1]) and np.all(m[:, 2] <= m[:, 3])
    assert np.any(m[:, 0] == m[:, 1]) or np.any(m[:, 0] > 63)        # some empty for all rows
    assert np.any((m[:, 0] <= 0) & (m[:, 1] >= 64))                   # some hide every row
    assert np.any((m[:, 0] > 0) & (m[:, 1] < 64))                     # some cut rows in the middle


def test_band_columns_are_the_band():
    for wl, wr in [(3, 0), (-1, 0), (2, 5), (-1, 4), (0, 0)]:
        m = masks.band(1, 20, wl, wr)[0, 0]
        vis = dense_visible(m, 20, False)
        i, j = np.meshgrid(np.arange(20), np.arange(20), indexing="ij")
        want = np.ones((20, 20), dtype=bool)
        if wl >= 0:
            want &= j >= i - wl
        if wr >= 0:
            want &= j <= i + wr
        assert np.array_equal(vis, want), (wl, wr)


def test_documents_are_block_diagonal():
    lens = [5, 1, 7, 3]
    m = masks.documents([lens], 16)[0, 0]
    doc = np.repeat(np.arange(len(lens)), lens)
    i, j = np.meshgrid(np.arange(16), np.arange(16), indexing="ij")
    assert np.array_equal(dense_visible(m, 16, True), (doc[i] == doc[j]) & (j <= i))
    mb = masks.documents([lens], 16, bidirectional=True)[0, 0]
    assert np.array_equal(dense_visible(mb, 16, False), doc[i] == doc[j])
    assert masks.visible_pairs(m[None, None], 16, True)[0, 0] == sum(n * (n + 1) // 2 for n in lens)


def test_prefix_lm():
    m = masks.prefix_lm(1, 12, 4)[0, 0]
    i, j = np.meshgrid(np.arange(12), np.arange(12), indexing="ij")
    assert np.array_equal(dense_visible(m, 12, False), (j < 4) | (j <= i))


def test_document_workload_flops_closed_form():
    """The document workload counts 4*d*H FLOPs per visible pair: for causal
    documents that is sum over documents of n(n+1)/2 pairs per batch entry."""
    from exact_attention_152_b200.workloads import WORKLOADS
    w = WORKLOADS["docs_b2h16n8k_d128_causal"]
    pairs = sum(n * (n + 1) // 2 for b in range(w.B) for n in w.doc_lengths(b))
    assert w.flops == 4.0 * w.d * w.H * pairs
    assert all(sum(w.doc_lengths(b)) == w.Nk for b in range(w.B))
    assert all(256 <= n <= 4096 for b in range(w.B) for n in w.doc_lengths(b)[:-1])


def test_block_summary_rules_are_sound():
    """The block summaries the kernels use decide two things per (128-key block,
    row range): 'every key hides every row' (max lo <= r0 and min hi >= r1 for
    one interval) lets a block be skipped, and 'no key's interval meets the
    rows' (max hi <= r0 or min lo >= r1 for both intervals) lets a warp skip
    element-wise masking.  Both must only fire when brute force agrees."""
    rng = np.random.default_rng(7)
    fired = {"hide_all": 0, "no_touch": 0}
    for trial in range(40):
        nq, nk = 300, 256
        m = masks.random_intervals(100 + trial, 1, 1, nq, nk)[0, 0].astype(np.int64)
        if trial % 3 == 0:  # documents too, where the rules fire often
            m = masks.documents([[70, 50, 90, 46]], nk)[0, 0].astype(np.int64)
        vis = dense_visible(m, nq, False)
        for blk in range(nk // 128):
            c = m[blk * 128:(blk + 1) * 128]
            e1, e2 = c[:, 0] >= c[:, 1], c[:, 2] >= c[:, 3]
            big, small = np.iinfo(np.int64).max, np.iinfo(np.int64).min
            lo1, hi1 = np.where(e1, big, c[:, 0]), np.where(e1, small, c[:, 1])
            lo2, hi2 = np.where(e2, big, c[:, 2]), np.where(e2, small, c[:, 3])
            for _ in range(10):
                r0 = int(rng.integers(0, nq - 1))
                r1 = int(rng.integers(r0 + 1, min(nq, r0 + 64) + 1))
                block = vis[r0:r1, blk * 128:(blk + 1) * 128]
                hide_all = (lo1.max() <= r0 and hi1.min() >= r1) or (lo2.max() <= r0 and hi2.min() >= r1)
                if hide_all:
                    assert not block.any()
                    fired["hide_all"] += 1
                touch = not (hi1.max() <= r0 or lo1.min() >= r1) or not (hi2.max() <= r0 or lo2.min() >= r1)
                if not touch:
                    assert block.all()
                    fired["no_touch"] += 1
    assert fired["hide_all"] > 0 and fired["no_touch"] > 0, fired


def test_backward_hidden_tile_ranges_are_sound():
    """The backward skips, per 128-key block, the query tiles t in
    [ceil(max lo / 128), (min hi >= Nq ? last : min hi // 128 - 1)] of each
    interval: every key of the block hides all rows of those tiles.  Key and
    query lengths that are not multiples of 128 leave a partial last key block
    (keys past Nk take no part in its summary) and a partial last query tile."""
    for nq, nk in ((700, 384), (650, 333), (513, 200), (129, 129)):
        for trial in range(24):
            if trial % 2:
                m = masks.random_intervals(200 + trial + nq, 1, 1, nq, nk)[0, 0].astype(np.int64)
            else:
                m = masks.documents([masks.document_lengths(300 + trial, nk, 30, 160)], nk,
                                    bidirectional=True)[0, 0].astype(np.int64)
            vis = dense_visible(m, nq, False)
            n_qtiles = (nq + 127) // 128
            fired = 0
            for blk in range((nk + 127) // 128):
                c = m[blk * 128:min(nk, (blk + 1) * 128)]
                for lo_col, hi_col in ((0, 1), (2, 3)):
                    empty = c[:, lo_col] >= c[:, hi_col]
                    lo = np.where(empty, np.iinfo(np.int64).max, c[:, lo_col]).max()
                    hi = np.where(empty, np.iinfo(np.int64).min, c[:, hi_col]).min()
                    first = 0 if lo <= 0 else -(-lo // 128)
                    last = n_qtiles - 1 if hi >= nq else hi // 128 - 1
                    for t in range(max(first, 0), min(last, n_qtiles - 1) + 1):
                        assert not vis[128 * t:min(128 * t + 128, nq), blk * 128:min(nk, (blk + 1) * 128)].any()
                        fired += 1
            if trial % 2 == 0 and nq >= 500:
                assert fired > 0, (nq, nk, trial)
