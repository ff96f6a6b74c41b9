"""Host layout builder vs the oracle's re-derivation from the explicit sets.

The library computes tiles from closed-form row intervals; the oracle walks
every live (i, j) pair. They must agree bit for bit: the same segments and
views, the same tiles in the same order, the same live counts and flags.
Runs on the CPU (host-only layouts, no CUDA call)."""
import ctypes

import numpy as np
import pytest

import factorized_sparse_self_b200 as st

CASES = [
    # kind, mode, T, l, c
    ("fixed", "split", 1024, 64, 8),
    ("fixed", "merged", 1536, 128, 8),
    ("fixed", "split", 768, 96, 4),
    ("fixed", "merged", 512, 64, 64),
    ("fixed", "merged", 640, 40, 5),        # c does not divide 128: natural-order summary keys
    ("fixed", "split", 384, 48, 16),
    ("strided", "split", 1536, 192, 1),
    ("strided", "merged", 2048, 256, 1),
    ("strided", "split", 1024, 16, 1),
    ("strided", "merged", 1024, 32, 1),
    ("strided", "split", 1024, 64, 1),      # P = 16: classes packed 8 to a tile
    ("strided", "merged", 512, 128, 1),     # P = 4: too short to pack, padded
    ("strided", "split", 3072, 32, 1),      # P = 96 does not divide 128: padded
    ("strided", "merged", 4096, 32, 1),     # P = 128: one class per tile
    ("strided", "merged", 1000, 48, 1),     # T not a multiple of l: no class view
    ("strided", "split", 384, 384, 1),      # l = T
    ("strided", "merged", 256, 1000, 1),    # l > T
    ("fixed", "split", 256, 300, 7),        # l > T
    ("dense", "merged", 640, 1, 1),
    ("dense", "merged", 200, 1, 1),         # ragged T
]


def _triples(ptr, idx, live, transpose):
    rows = np.repeat(np.arange(len(ptr) - 1), np.diff(ptr))
    if transpose:
        return idx.astype(np.int64), rows.astype(np.int64), live.astype(np.int64)
    return rows.astype(np.int64), idx.astype(np.int64), live.astype(np.int64)


@pytest.mark.parametrize("case", CASES)
def test_layout_bit_exact_vs_oracle(orc, case):
    kind, mode, T, l, c = case
    L = st.st_pattern_layout_host(kind, mode, T, l, c)
    nhc, nseg = L.counts()
    assert nhc == orc.num_head_classes(kind, mode)
    assert nseg == orc.num_segments(kind, mode)
    for hc in range(nhc):
        total = 0
        for seg in list(range(nseg)) + [-1]:
            if seg >= 0:
                qv, kv, _ = L.segment_info(hc, seg)
                assert (qv, kv) == orc.segment_views(kind, mode, T, l, c, hc, seg)
            oq, ok, olive = orc.layout_tiles(kind, mode, T, l, c, hc, seg)
            ptr, idx, flags, live = L.export(hc, seg, transpose=False)
            q, k, lv = _triples(ptr, idx, live, False)
            np.testing.assert_array_equal(q, oq)
            np.testing.assert_array_equal(k, ok)
            np.testing.assert_array_equal(lv, olive)
            np.testing.assert_array_equal(flags, (olive != 128 * 128).astype(np.uint8))
            # the CSC export lists the same tiles, key-major
            ptr_t, idx_t, flags_t, live_t = L.export(hc, seg, transpose=True)
            q2, k2, lv2 = _triples(ptr_t, idx_t, live_t, True)
            order = np.lexsort((oq, ok))
            np.testing.assert_array_equal(q2, oq[order])
            np.testing.assert_array_equal(k2, ok[order])
            np.testing.assert_array_equal(lv2, olive[order])
            if seg >= 0:
                total += int(live.sum())
        h = hc if mode == "split" else 0
        assert total == L.nnz(hc) == orc.nnz(kind, mode, T, l, c, h)


def test_gathered_views_make_tiles_dense(orc):
    """The gather views are what make the live tiles dense: tile efficiency of
    the segment tilings vs the plain natural tiling, text-like fixed pattern."""
    L = st.st_pattern_layout_host("fixed", "merged", 12288, 128, 8)
    live_seg = sum(int(L.export(0, s)[3].sum()) for s in range(2))
    area_seg = sum(len(L.export(0, s)[1]) for s in range(2)) * 128 * 128
    _, idx, _, live_nat = L.export(0, -1)
    eff_seg = live_seg / area_seg
    eff_nat = live_nat.sum() / (len(idx) * 128 * 128)
    assert live_seg == live_nat.sum() == 5462016
    assert eff_seg > 0.75 and eff_nat < 0.08


def test_invalid_descriptors_rejected():
    for args in [("fixed", "split", 256, 16, 0), ("fixed", "split", 256, 16, 17),
                 ("strided", "split", 256, 0, 1), ("strided", "split", 0, 4, 1),
                 (7, "split", 256, 16, 1), ("strided", 5, 256, 16, 1)]:
        with pytest.raises(st.StatusError) as e:
            st.st_pattern_layout_host(*args)
        assert e.value.code == st.ST_ERR_INVALID


def _golden_tiles():
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "layout_tiles.json")
    with open(path) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _golden_tiles(),
                         ids=lambda c: f"{c['kind']}-{c['mode']}-T{c['T']}-l{c['l']}-"
                                       f"hc{c['head_class']}-seg{c['segment']}")
def test_tile_coordinates_match_hand_derived_lists(orc, case):
    """Pins the tile coordinates of the summary and residue-class orders: the
    oracle's pair-by-pair tiling and the library's export must both give the
    hand-derived (query tile, key tile, live) lists, not only the right totals."""
    want = np.array(case["tiles"], dtype=np.int64)
    args = (case["kind"], case["mode"], case["T"], case["l"], case["c"])
    hc, seg = case["head_class"], case["segment"]
    oq, ok, olive = orc.layout_tiles(*args, hc, seg)
    np.testing.assert_array_equal(np.stack([oq, ok, olive], axis=1), want)
    L = st.st_pattern_layout_host(*args)
    ptr, idx, flags, live = L.export(hc, seg, transpose=False)
    q, k, lv = _triples(ptr, idx, live, False)
    np.testing.assert_array_equal(np.stack([q, k, lv], axis=1), want)
    np.testing.assert_array_equal(flags, (want[:, 2] != 128 * 128).astype(np.uint8))


# Which gradient rows the 16-bit backward zero-fills or accumulates in fp32
# (st_layout_rows), against the sets themselves: the membership rule of the
# oracle's numpy restatement, brute force over all (i, j) of one head.
ROW_CASES = [
    ("fixed", "merged", 1536, 128, 8),
    ("fixed", "merged", 1024, 32, 16),
    ("fixed", "merged", 2048, 256, 16),
    ("fixed", "merged", 1536, 48, 8),
    ("fixed", "split", 1024, 64, 8),
    ("strided", "split", 1536, 192, 1),
    ("strided", "merged", 2048, 256, 1),
]


@pytest.mark.parametrize("case", ROW_CASES, ids=lambda c: "-".join(map(str, c)))
def test_gradient_row_lists_follow_the_sets(case):
    from oracle import reference_np as ref
    kind, mode, T, l, c = case
    L = st.st_pattern_layout_host(kind, mode, T, l, c)
    n_hc = L.counts()[0]
    for hc in range(n_hc):
        m = ref.mask(kind, mode, T, l, c, hc)  # head hc has the class's parity
        q_empty = set(np.flatnonzero(~m.any(axis=1)).tolist())
        k_unused = set(np.flatnonzero(~m.any(axis=0)).tolist())
        q_acc, k_acc = L.rows(hc, L.ROWS_Q_ACC), L.rows(hc, L.ROWS_K_ACC)
        q_zero, k_zero = L.rows(hc, L.ROWS_Q_ZERO), L.rows(hc, L.ROWS_K_ZERO)
        for r in (q_acc, k_acc, q_zero, k_zero):
            assert np.all(np.diff(r) > 0) and (r.size == 0 or (r[0] >= 0 and r[-1] < T))
        # a zero-filled row must have a zero gradient: no live pair at all
        assert set(q_zero.tolist()) <= q_empty
        assert set(k_zero.tolist()) <= k_unused
        assert not set(q_zero.tolist()) & set(q_acc.tolist())
        assert not set(k_zero.tolist()) & set(k_acc.tolist())
    if kind == "fixed" and mode == "split":
        # the summary heads read summary keys only: every other key row is
        # zero-filled, and no summary key is
        summary = np.flatnonzero(np.arange(T) % l >= l - c)
        assert set(L.rows(1, L.ROWS_K_ZERO).tolist()) == set(range(T)) - set(summary.tolist())
        assert L.rows(0, L.ROWS_K_ACC).size == 0  # block heads: one unit per key tile
    if kind == "fixed" and mode == "merged":
        summary = np.flatnonzero(np.arange(T) % l >= l - c)
        if (128 % l == 0 and c * (128 // l) <= 64) or (l % 128 == 0 and c <= 64):
            # block key tiles are stored directly and add only their summary
            # rows: exactly the summary keys accumulate
            assert np.array_equal(L.rows(0, L.ROWS_K_ACC), summary)
        else:
            # l does not divide 128: every block tile holds summary keys and
            # accumulates as a whole
            assert np.array_equal(L.rows(0, L.ROWS_K_ACC), np.arange(T))
    if mode == "merged" or kind == "strided":
        # causal sets are never empty: no dQ row is zero-filled
        for hc in range(n_hc):
            assert L.rows(hc, L.ROWS_Q_ZERO).size == 0


def test_row_list_arguments():
    L = st.st_pattern_layout_host("fixed", "merged", 1536, 128, 8)
    with pytest.raises(st.StatusError):
        L.rows(1, 0)  # one head class
    with pytest.raises(st.StatusError):
        L.rows(0, 4)
    n = ctypes.c_int64(3)
    buf = (ctypes.c_int32 * 3)()
    assert st.lib().st_layout_rows(L.handle, 0, 1, buf, ctypes.byref(n)) == st.ST_ERR_WORKSPACE
    assert n.value == 96  # 12 blocks x 8 summary keys, reported despite the short buffer
