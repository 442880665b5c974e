"""Pins of the oracle's bank-balanced word order (v2) for 64 x 64 tiles: the
Flash-LLM review's ahead-of-time, bank-conflict-aware reordering of each
tile's NonZeros (section 3), restated for the 128-byte swizzled dense tile the
B200 kernel expands into.  v2 changes only the order of a tile's words, so
everything the ascending-loc encoding fixes (offsets, the set of words,
padding, the decoded matrix) must be unchanged; the rule's own guarantees are
checked as properties, a few tiles against hand-derived orders, and the
effect against the quantity it exists to reduce (bank wavefronts per 32-word
store window)."""
import json
from pathlib import Path

import numpy as np
import pytest

import oracle
import synth

GOLDEN = json.loads((Path(__file__).parent / "golden" / "tcsl_v2_order.json").read_text())
SENT = 0xFFFF0000


def _tile_words(off, words, t):
    seg = words[off[t]:off[t + 1]]
    real = seg[seg != SENT]
    assert (seg[len(real):] == SENT).all()  # sentinels only after the real words
    return real


def _wavefronts(locs):
    """Bank wavefronts of one warp-wide 16-bit store of these locs: the largest
    number of distinct 32-bit words that fall in one bank."""
    x = 2 * locs.astype(np.int64)
    off = x ^ ((x >> 3) & 0x70)
    w32 = off >> 2
    per_bank = {}
    for b, a in set(zip((w32 & 31).tolist(), w32.tolist())):
        per_bank[b] = per_bank.get(b, 0) + 1
    return max(per_bank.values())


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=[c["name"] for c in GOLDEN["cases"]])
def test_golden_orders(case):
    A = np.zeros((64, 64), dtype=np.float16)
    for i, loc in enumerate(case["locs"]):
        A[loc // 64, loc % 64] = np.float16(i + 1)
    off, w, _ = oracle.tcsl_encode(A, order=1)
    got = (_tile_words(off, w, 0) >> 16).tolist()
    assert got == case["v2_locs"]


@pytest.mark.parametrize("s_pct,structure", [(50, "uniform"), (80, "uniform"), (90, "row_magnitude"),
                                             (95, "column_clustered"), (70, "power_law"), (0, "uniform")])
def test_v2_is_a_reordering_with_the_rule_properties(s_pct, structure):
    W = synth.sparse_weight(320, 448, s_pct, structure, (230, s_pct))  # ragged: 5 x 7 tiles
    o1, w1, n1 = oracle.tcsl_encode(W)
    o2, w2, n2 = oracle.tcsl_encode(W, order=1)
    assert np.array_equal(o1, o2) and n1 == n2
    assert np.array_equal(oracle.tcsl_decode(o2, w2, *W.shape), W.view(np.uint16))
    for t in range(len(o1) - 1):
        a = _tile_words(o1, w1, t)
        b = _tile_words(o2, w2, t)
        assert np.array_equal(np.sort(a), np.sort(b))           # same words, same count
        locs = (b >> 16).astype(np.int64)
        banks = oracle.bank_of_loc(locs)
        for bk in np.unique(banks):                              # each bank in ascending loc
            assert np.all(np.diff(locs[banks == bk]) > 0)
        for s in range(0, len(b), 32):                           # distinct banks per window
            left = np.bincount(banks[s:], minlength=32)
            win = banks[s:s + 32]
            assert len(np.unique(win)) == min(len(win), int((left > 0).sum()))


def test_v2_cuts_store_wavefronts_on_the_workload_matrices():
    for s_pct, want in ((70, 1.5), (80, 1.6), (90, 1.8)):
        W = synth.sparse_weight(512, 1024, s_pct, "uniform", (231, s_pct))
        per = []
        for order in (0, 1):
            off, w, _ = oracle.tcsl_encode(W, order=order)
            tot = n = 0
            for t in range(len(off) - 1):
                locs = (_tile_words(off, w, t) >> 16).astype(np.int64)
                for s in range(0, len(locs), 32):
                    tot += _wavefronts(locs[s:s + 32])
                    n += 1
            per.append(tot / n)
        assert per[1] < 0.7 * per[0] and per[1] < want, (s_pct, per)


def test_v2_needs_64x64_tiles():
    with pytest.raises(Exception):
        oracle.tcsl_encode(np.ones((64, 64), dtype=np.float16), tile_m=32, tile_k=64, order=1)
