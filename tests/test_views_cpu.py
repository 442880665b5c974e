"""Row and K-range views of a Tiled-CSL matrix (TCSL.slice_rows / slice_cols),
checked on the host: a view addresses tile (i, j) at tile_offsets[i * ld + j]
(the rule the SpMM kernel and the partition kernel use), so gathering a view's
tiles through that rule must give exactly the oracle's encoding of the same
rows and columns encoded on their own.  No device is needed: the views are
pointer arithmetic over the full matrix's offsets."""
import numpy as np
import pytest
import torch

import oracle
import synth
from unstructured_sparse_skinny_b200.binding import TCSL


def _full(M, K, s_pct=80, structure="power_law", key=(250, 0)):
    W = synth.sparse_weight(M, K, s_pct, structure, key)
    off, words, nnz = oracle.tcsl_encode(W)
    return W, TCSL(torch.from_numpy(off), torch.from_numpy(words.view(np.int32)), nnz, M, K), words


def _gather(view, words):
    """The view's tiles, in its own row-major tile order, through its addressing rule."""
    TM, TK = -(-view.M // 64), -(-view.K // 64)
    off, ld = view.tile_offsets.numpy(), view.ld
    segs = [words[off[i * ld + j]:off[i * ld + j + 1]] for i in range(TM) for j in range(TK)]
    g_off = np.concatenate([[0], np.cumsum([len(s) for s in segs])]).astype(np.int32)
    g_words = np.concatenate(segs) if segs else np.zeros(0, np.uint32)
    return g_off, g_words


def _assert_same(view, words, W_sub):
    g_off, g_words = _gather(view, words)
    s_off, s_words, _ = oracle.tcsl_encode(np.ascontiguousarray(W_sub))
    assert np.array_equal(g_off, s_off)
    assert g_words.tobytes() == s_words.tobytes()


@pytest.mark.parametrize("k0,k1", [(0, 64), (64, 640), (576, 968), (960, 968), (0, 968), (128, 192)])
def test_k_range_view_addresses_its_tiles(k0, k1):
    W, t, words = _full(330, 968)
    v = t.slice_cols(k0, k1)
    assert (v.M, v.K, v.ld, v.nnz, v.piece_bounds) == (330, k1 - k0, 16, -1, None)
    _assert_same(v, words, W[:, k0:k1])


@pytest.mark.parametrize("r0,r1", [(0, 64), (64, 330), (320, 330), (128, 256)])
def test_row_view_addresses_its_tiles(r0, r1):
    W, t, words = _full(330, 968)
    v = t.slice_rows(r0, r1)
    assert (v.M, v.K, v.ld) == (r1 - r0, 968, 16)
    _assert_same(v, words, W[r0:r1])


@pytest.mark.parametrize("rows,cols", [((64, 330), (128, 968)), ((0, 192), (64, 128)), ((256, 330), (960, 968))])
def test_views_compose_either_way(rows, cols):
    W, t, words = _full(330, 968, 70, "column_clustered", (251, 0))
    a = t.slice_cols(*cols).slice_rows(*rows)
    b = t.slice_rows(*rows).slice_cols(*cols)
    for v in (a, b):
        _assert_same(v, words, W[rows[0]:rows[1], cols[0]:cols[1]])


@pytest.mark.parametrize("bad", [(1, 64), (0, 100), (64, 64), (-64, 64), (0, 1032)])
def test_k_range_view_rejects_unaligned_ranges(bad):
    _, t, _ = _full(128, 968)
    with pytest.raises(ValueError):
        t.slice_cols(*bad)


@pytest.mark.parametrize("bad", [(1, 64), (0, 100), (64, 64), (0, 200)])
def test_row_view_rejects_unaligned_ranges(bad):
    _, t, _ = _full(130, 256)
    with pytest.raises(ValueError):
        t.slice_rows(*bad)


def test_view_struct_carries_ld_and_table():
    _, t, _ = _full(256, 512)
    v = t.slice_cols(128, 384).view()
    assert v.offsets_ld == 8 and v.K == 256 and v.nnz == -1
    assert v.piece_bounds is None and v.bounds_pieces == 0 and v.reserved == 0
    assert t.view().offsets_ld == 0 and t.ld == 8
