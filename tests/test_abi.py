"""Host-side checks of the C ABI: the library loads, exports every function
include/ba.h declares, rejects invalid problems before launching anything,
and its planner matches a Python restatement of the zigzag row tiling.
No GPU needed."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import oracle as orc
import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ba():
    from branch_attention_speculative_packed_b200 import build
    build.build()
    import branch_attention_speculative_packed_b200 as m
    return m


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"BA_API\s+[\w\s\*]+?\b(ba_\w+)\s*\(", txt)
    return sorted(set(names))


def test_library_exports_every_declared_symbol(ba):
    declared = _declared()
    assert "ba_fused_fwd" in declared and "ba_bwd" in declared
    L = ba.lib()
    for name in declared:
        assert hasattr(L, name), name
    assert sorted(ba.EXPORTED) == sorted(declared) or set(ba.EXPORTED) <= set(declared)


def test_status_strings(ba):
    for s in (0, -1, -2, -3, -4, -5):
        assert isinstance(ba.status_string(s), str) and ba.status_string(s)


def _attn(ba, cu, anc, **kw):
    args = dict(Hq=4, Hkv=2, d=128, B=3, mode=0, R=2, device="cpu")
    args.update(kw)
    return ba.BranchAttention(cu, anc, **args)


@pytest.mark.parametrize("bad", [
    dict(cu=[0, 5, 5, 10], anc=[1]),          # empty document
    dict(cu=[0, 6, 4, 10], anc=[1]),          # decreasing
    dict(cu=[1, 5, 10], anc=[1]),             # does not start at 0
    dict(cu=[0, 5, 10], anc=[3, 2]),          # anchors not ascending
    dict(cu=[0, 5, 10], anc=[10]),            # anchor out of range
    dict(cu=[0, 5, 10], anc=[-1]),            # negative anchor
    dict(cu=[0, 5, 10], anc=[1], Hq=3),       # Hq % Hkv != 0
    dict(cu=[0, 5, 10], anc=[1], R=0),        # no ranks
    dict(cu=[0, 5, 10], anc=[1], R=65),       # too many ranks
    dict(cu=[0, 5, 10], anc=[1], B=0),        # empty branches
    dict(cu=[0, 5, 10], anc=[1], mode=2),     # unknown mask
    dict(cu=[0, 5, 10], anc=[1], d=96),       # unsupported head dim
])
def test_invalid_problems_rejected(ba, bad):
    bad = dict(bad)
    cu, anc = bad.pop("cu"), bad.pop("anc")
    a = _attn(ba, cu, anc, **bad)
    with pytest.raises(ValueError):
        a.workspace_size(ba.BA_WS_FWD)
    with pytest.raises(ba.BAError):
        a.plan_stats()


def test_duplicate_anchors_accepted(ba):
    a = _attn(ba, [0, 5, 10], [2, 2, 7])
    assert a.workspace_size(ba.BA_WS_FWD) > 0


# ---------------------------------------------------------------------------
# planner restated in Python
# ---------------------------------------------------------------------------

def _restated_plan(cu, anc, B, R):
    """Row tiles per document: the document's rows sorted by (limit,
    main-before-branch, branch index, depth), cut into 128-row tiles; a tile
    visits the main key tiles [doc start, max limit] in steps of 128 and is
    owned by the zigzag rank of the chunk holding its first row."""
    cu = list(cu)
    anc = list(anc)
    tiles = 0
    pairs = 0
    rank_pairs = [0] * R
    chunks = orc.zigzag_chunks(np.array(cu), R)
    for di in range(len(cu) - 1):
        s, e = cu[di], cu[di + 1]
        rows = [(p, 0, 0, 0) for p in range(s, e)]
        rows += [(a, 1, b, t) for b, a in enumerate(anc) if s <= a < e for t in range(B)]
        rows.sort()
        for i in range(0, len(rows), 128):
            tile = rows[i:i + 128]
            tiles += 1
            n = -(-(tile[-1][0] - s + 1) // 128)
            pairs += n
            first = tile[0][0]
            owner = [c[4] for c in chunks if c[0] == di and c[2] <= first < c[3]][0]
            rank_pairs[owner] += n
    return tiles, pairs, rank_pairs


@pytest.mark.parametrize("case", [
    ([0, 256], [23, 43, 60, 72, 179, 200, 201, 255], 4, 2),
    ([0, 3, 10, 700, 1000], list(range(0, 1000, 7)), 3, 4),
    ([0, 1, 2, 3], [0, 1, 2], 2, 8),           # documents shorter than 2R
    ([0, 500], [], 3, 3),                     # no branches
    ([0, 300, 301], [299, 299, 300], 16, 1),  # duplicate anchors, anchor on 1-token doc
])
def test_planner_matches_restatement(ba, case):
    cu, anc, B, R = case
    a = _attn(ba, cu, anc, B=B, R=R)
    st = a.plan_stats()
    t, p, rp = _restated_plan(cu, anc, B, R)
    assert st["row_tiles"] == t
    assert st["tile_pairs"] == p
    assert a.rank_work() == rp
    assert st["visible_pairs"] == orc.visible_pair_count(np.array(cu), np.array(anc), B, 0)


@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_planner_on_workload_layouts(ba, idx):
    cfg = wl.CONFIGS[idx]
    cu, anc = wl.make_layout(idx)
    a = ba.BranchAttention(cu, anc, Hq=cfg.Hq, Hkv=cfg.Hkv, d=cfg.d, B=cfg.B, mode=cfg.mode,
                           R=cfg.R, device="cpu")
    st = a.plan_stats()
    assert st["visible_pairs"] == orc.visible_pair_count(cu.numpy(), anc.numpy(), cfg.B, cfg.mode)
    if idx <= 2:
        t, p, rp = _restated_plan(cu.tolist(), anc.tolist(), cfg.B, cfg.R)
        assert (st["row_tiles"], st["tile_pairs"]) == (t, p)
        assert a.rank_work() == rp
        assert a.fwd_pairs() == _restated_pairs(cu.tolist(), anc.tolist(), cfg.B)
    # every visible pair lies in a visited tile pair
    assert st["tile_pairs"] * 128 * 128 >= st["visible_pairs"] - cfg.n_anchors * cfg.B * cfg.B


def _restated_pairs(cu, anc, B):
    """Forward work items restated: per document, tiles 2k and 2k+1 (the last
    alone when the count is odd); a tile costs its main key tiles plus its
    branch key tiles (the branches with a row in the tile, B keys each); a pair
    costs both minus the shorter main range they share; most cost first,
    position order among equals."""
    tiles = []  # (doc, main key tiles, branch key tiles)
    for di in range(len(cu) - 1):
        s, e = cu[di], cu[di + 1]
        rows = [(p, 0, 0, 0) for p in range(s, e)]
        rows += [(a, 1, b, t) for b, a in enumerate(anc) if s <= a < e for t in range(B)]
        rows.sort()
        for i in range(0, len(rows), 128):
            tile = rows[i:i + 128]
            nkv = -(-(tile[-1][0] - s + 1) // 128)
            bs = [r[2] for r in tile if r[1] == 1]
            nbr = -(-((max(bs) - min(bs) + 1) * B) // 128) if bs else 0
            tiles.append((di, nkv, nbr))
    pairs, cost = [], []
    i = 0
    while i < len(tiles):
        two = i + 1 < len(tiles) and tiles[i + 1][0] == tiles[i][0]
        c = tiles[i][1] + tiles[i][2]
        if two:
            c += tiles[i + 1][1] + tiles[i + 1][2] - min(tiles[i][1], tiles[i + 1][1])
        pairs.append((i, i + 1 if two else -1))
        cost.append(c)
        i += 2 if two else 1
    order = sorted(range(len(pairs)), key=lambda k: -cost[k])  # stable
    return [pairs[k] for k in order]


@pytest.mark.parametrize("case", [
    ([0, 256], [23, 43, 60, 72, 179, 200, 201, 255], 4, 2),
    ([0, 3, 10, 700, 1000], list(range(0, 1000, 7)), 3, 4),
    ([0, 1, 2, 3], [0, 1, 2], 2, 8),
    ([0, 500], [], 3, 3),
    ([0, 300, 301], [299, 299, 300], 16, 1),
])
def test_forward_pairs_match_restatement(ba, case):
    cu, anc, B, R = case
    a = _attn(ba, cu, anc, B=B, R=R)
    got = a.fwd_pairs()
    assert got == _restated_pairs(cu, anc, B)
    covered = sorted(t for p in got for t in p if t >= 0)
    assert covered == list(range(a.plan_stats()["row_tiles"]))  # every tile exactly once


@pytest.mark.parametrize("R", [2, 4, 8])
def test_zigzag_split_balances_causal_work(ba, R):
    """Rank r owns chunks r and 2R-1-r, so every rank gets the same share of
    the triangular causal work (up to tile rounding): the load-balancing the
    pages attribute to the zigzag split.  A contiguous split would give the
    last rank about 2R-1 times the first rank's work."""
    L = 65536
    a = _attn(ba, [0, L, 2 * L], list(range(0, 2 * L, 3)), B=3, R=R)
    w = a.rank_work()
    assert len(w) == R and sum(w) == a.plan_stats()["tile_pairs"]
    assert max(w) / min(w) < 1.05, w


def test_plan_cache_reuses_and_clears(ba):
    """A second call with identical sizes and packing contents reuses the
    cached plan; a different packing (same sizes) misses; ba_clear_cache drops
    every entry, after which the same problem plans again."""
    ba.clear_cache()
    assert ba.plan_cache_stats()["entries"] == 0
    a = _attn(ba, [0, 300, 700], [5, 299, 301, 650])
    s0 = ba.plan_cache_stats()
    first = a.plan_stats()
    s1 = ba.plan_cache_stats()
    assert (s1["misses"], s1["hits"], s1["entries"]) == (s0["misses"] + 1, s0["hits"], 1)
    assert a.plan_stats() == first
    a.workspace_size(ba.BA_WS_BWD)  # forward and backward share the entry
    s2 = ba.plan_cache_stats()
    assert (s2["misses"], s2["hits"], s2["entries"]) == (s1["misses"], s1["hits"] + 2, 1)
    # same sizes, different anchor contents: a different plan
    b = _attn(ba, [0, 300, 700], [5, 299, 302, 650])
    b.plan_stats()
    s3 = ba.plan_cache_stats()
    assert (s3["misses"], s3["entries"]) == (s2["misses"] + 1, 2)
    assert a.prepare() >= 0.0
    ba.clear_cache()
    assert ba.plan_cache_stats()["entries"] == 0
    assert a.plan_stats() == first
    s4 = ba.plan_cache_stats()
    assert s4["misses"] == s3["misses"] + 1 and s4["entries"] == 1
    ba.clear_cache()


def test_plan_cache_keeps_the_16_most_recent(ba):
    ba.clear_cache()
    probs = [_attn(ba, [0, 100 + i], [i]) for i in range(20)]
    for p in probs:
        p.plan_stats()
    assert ba.plan_cache_stats()["entries"] == 16
    before = ba.plan_cache_stats()
    probs[-1].plan_stats()   # most recent: still cached
    assert ba.plan_cache_stats()["hits"] == before["hits"] + 1
    probs[0].plan_stats()    # least recent: evicted, plans again
    assert ba.plan_cache_stats()["misses"] == before["misses"] + 1
    ba.clear_cache()


def test_visible_pairs_with_window_and_bitmask_match_oracle_count(ba):
    """The planner's exact pair count under a main-prefix window and under
    per-branch mask words equals the oracle's counting rule."""
    rs = np.random.default_rng(0)
    for trial in range(40):
        S = int(rs.integers(1, 400))
        nd = int(rs.integers(1, min(S, 6) + 1))
        cuts = sorted(rs.choice(np.arange(1, S), nd - 1, replace=False).tolist()) if nd > 1 else []
        cu = [0] + cuts + [S]
        anc = sorted(rs.integers(0, S, int(rs.integers(0, S + 1))).tolist())
        B = int(rs.integers(1, 9))
        mode = int(rs.integers(0, 3))
        W = int(rs.choice([0, 1, 3, 17, 500]))
        bm = rs.integers(0, 2 ** B, size=(len(anc), B), dtype=np.uint64) if mode == 2 else None
        a = ba.BranchAttention(cu, anc, Hq=2, Hkv=1, d=64, B=B, mode=mode, R=int(rs.integers(1, 9)),
                               device="cpu", window=W, branch_mask=bm)
        exp = orc.visible_pair_count(np.array(cu), np.array(anc, dtype=np.int64), B, mode, window=W,
                                     branch_mask=bm)
        assert a.plan_stats()["visible_pairs"] == exp, (trial, mode, W)


def test_bitmask_mode_needs_its_words(ba):
    a = ba.BranchAttention([0, 10], [3], Hq=2, Hkv=1, d=64, B=2, mode=2, device="cpu")
    with pytest.raises(ba.BAError):
        a.plan_stats()


def test_one_rank_plans_partition_the_rows(ba):
    """The plans of the R virtual ranks' rows (cp_rank) split the work: their
    visible-pair counts add up to the whole problem's, each rank's pairs are
    within a few percent of the mean for long documents (the zigzag balance),
    and an out-of-range rank is refused."""
    rs = np.random.default_rng(3)
    for trial in range(12):
        S = int(rs.integers(2, 3000))
        nd = int(rs.integers(1, min(S, 5) + 1))
        cuts = sorted(rs.choice(np.arange(1, S), nd - 1, replace=False).tolist()) if nd > 1 else []
        cu = [0] + cuts + [S]
        anc = sorted(rs.integers(0, S, int(rs.integers(0, S + 1))).tolist())
        R = int(rs.integers(1, 9))
        W = int(rs.choice([0, 50]))
        kw = dict(Hq=2, Hkv=1, d=64, B=3, mode=0, R=R, device="cpu", window=W)
        whole = ba.BranchAttention(cu, anc, **kw).plan_stats()["visible_pairs"]
        parts = [ba.BranchAttention(cu, anc, cp_rank=r, **kw).plan_stats()["visible_pairs"] for r in range(R)]
        assert sum(parts) == whole, (trial, parts, whole)
    big = [ba.BranchAttention([0, 65536], list(range(65536)), Hq=1, Hkv=1, d=64, B=3, mode=0, R=8,
                              device="cpu", cp_rank=r).plan_stats()["visible_pairs"] for r in range(8)]
    assert max(big) / min(big) < 1.01
    with pytest.raises(ba.BAError):
        ba.BranchAttention([0, 10], [1], Hq=1, Hkv=1, d=64, B=1, mode=0, R=2, device="cpu",
                           cp_rank=2).plan_stats()
