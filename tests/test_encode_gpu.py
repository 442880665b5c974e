"""GPU Tiled-CSL encoder vs the oracle's encoder: offsets and words must be
byte-identical (Flash-LLM review, section 3, "sparse encoding format:
Tiled-CSL"), on every mask structure, ragged shapes, other tile sizes and
special fp16 bit patterns; plus the checked-mode validator."""
import numpy as np
import pytest
import torch

import oracle
import synth
import unstructured_sparse_skinny_b200 as fs
from tests.helpers import assert_encode_bit_exact, gpu_encode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("structure", ["uniform", "row_magnitude", "power_law", "column_clustered"])
@pytest.mark.parametrize("s_pct", [50, 80, 95])
def test_structures_bit_exact(structure, s_pct):
    W = synth.sparse_weight(1024, 1536, s_pct, structure, (100, 1))
    assert_encode_bit_exact(W)


@pytest.mark.parametrize("M,K,tm,tk", [(200, 136, 64, 64), (130, 72, 64, 64), (1, 8, 64, 64), (64, 64, 64, 64),
                                       (333, 264, 128, 64), (77, 40, 16, 8), (300, 512, 255, 256),
                                       (96, 96, 1, 8), (2048, 8, 64, 64), (8, 4096, 64, 64)])
def test_ragged_and_tile_sizes(M, K, tm, tk):
    g = np.random.default_rng(M + K)
    W = (g.standard_normal((M, K)) * 0.02).astype(np.float16)
    W[g.random((M, K)) < 0.7] = 0
    assert_encode_bit_exact(W, tm, tk)


def test_special_bit_patterns():
    g = np.random.default_rng(5)
    bits = (g.standard_normal((256, 512)) * 0.02).astype(np.float16).view(np.uint16)
    pick = g.random(bits.shape)
    bits[pick < 0.5] = 0
    bits[(pick >= 0.5) & (pick < 0.52)] = 0x8000   # -0.0 is stored
    bits[(pick >= 0.52) & (pick < 0.53)] = 0x7E01  # NaN payload
    bits[(pick >= 0.53) & (pick < 0.54)] = 0x7C00  # +Inf
    bits[(pick >= 0.54) & (pick < 0.55)] = 0x0001  # smallest subnormal
    t, off, words = assert_encode_bit_exact(bits.view(np.float16))
    assert np.array_equal(oracle.tcsl_decode(off, words, 256, 512), bits)


def test_empty_dense_and_single_entries():
    assert_encode_bit_exact(np.zeros((256, 256), dtype=np.float16))
    assert_encode_bit_exact(np.ones((192, 128), dtype=np.float16))
    W = np.zeros((128, 128), dtype=np.float16)
    W[0, 0] = 1
    W[63, 63] = -2
    W[127, 64] = 3
    assert_encode_bit_exact(W)


def test_empty_matrix_shapes():
    t = gpu_encode(np.zeros((0, 64), dtype=np.float16))
    assert t.tile_offsets.cpu().tolist() == [0] and t.nwords == 0 and t.nnz == 0
    t = gpu_encode(np.zeros((64, 0), dtype=np.float16))
    assert t.tile_offsets.cpu().tolist() == [0]


def test_validate_accepts_and_rejects():
    W = synth.sparse_weight(512, 512, 80, "uniform", (100, 2))
    t = gpu_encode(W)
    fs.tcsl_validate(t)  # a fresh encoding is valid
    words = t.words.clone()
    corruptions = []
    w = words.clone(); w[5] = int(np.int32(np.uint32(0x3C00 | (4096 << 16)).view(np.int32)))  # loc out of tile
    corruptions.append(("loc", t.tile_offsets, w))
    w = words.clone(); w[1] = words[0].item()  # one location stored twice in a tile
    corruptions.append(("duplicate", t.tile_offsets, w))
    off = t.tile_offsets.clone(); off[3] += 2  # offset not a multiple of 4
    corruptions.append(("offset", off, words))
    w = words.clone(); w[5] = int(np.uint32(0xFFFF3C00).view(np.int32))  # sentinel location with value bits
    corruptions.append(("sentinel", t.tile_offsets, w))
    w = words.clone(); w[5] = int(words[5].item()) & ~0xFFFF  # a real word whose value bits are zero
    corruptions.append(("zero value", t.tile_offsets, w))
    for name, o, w in corruptions:
        bad = fs.TCSL(o, w, t.nnz, t.M, t.K)
        with pytest.raises(fs.FlashSpmmError) as e:
            fs.tcsl_validate(bad)
        assert e.value.status == 6, name
    fs.tcsl_validate(t)  # status word was cleared by the failing reads


# ---- word order v2 (bank-balanced), the page's ahead-of-time reorder restated for the B200 tile

def _v2_bit_exact(W):
    t = fs.tcsl_encode(torch.from_numpy(np.ascontiguousarray(W)).cuda(), order=1)
    fs.check_device_status()
    off, words, nnz = oracle.tcsl_encode(W, order=1)
    assert np.array_equal(t.tile_offsets.cpu().numpy(), off)
    gw = t.words.cpu().numpy().view(np.uint32)
    assert gw.size == words.size and gw.tobytes() == words.tobytes()
    assert t.nnz == nnz and t.order == 1
    return t


V2_CASES = [(st, s) for st in ("uniform", "row_magnitude", "power_law", "column_clustered")
            for s in (0, 50, 70, 80, 90, 99)
            if not (st == "power_law" and not 40 <= s <= 98)]  # power-law row densities lie in [2 %, 60 %]


@pytest.mark.parametrize("structure,s_pct", V2_CASES)
def test_v2_structures_bit_exact(structure, s_pct):
    W = synth.sparse_weight(768, 1024, s_pct, structure, (101, s_pct))
    _v2_bit_exact(W)


@pytest.mark.parametrize("M,K", [(200, 136), (130, 72), (1, 8), (64, 64), (2048, 8), (8, 4096), (333, 1000)])
def test_v2_ragged(M, K):
    g = np.random.default_rng(M * 7 + K)
    W = (g.standard_normal((M, K)) * 0.02).astype(np.float16)
    W[g.random((M, K)) < 0.75] = 0
    _v2_bit_exact(W)


def test_v2_edge_tiles():
    _v2_bit_exact(np.zeros((128, 192), dtype=np.float16))          # empty tiles
    _v2_bit_exact(np.ones((128, 128), dtype=np.float16))           # 4096-word tiles, one bank order
    W = np.zeros((128, 128), dtype=np.float16)
    W[:, 0] = 1                                                   # every word in the same two banks
    W[5, 7] = 2
    _v2_bit_exact(W)


def test_v2_validates_and_keeps_decode():
    W = synth.sparse_weight(1024, 1024, 80, "power_law", (102, 0))
    t = _v2_bit_exact(W)
    fs.tcsl_validate(t)
    off = t.tile_offsets.cpu().numpy()
    assert np.array_equal(oracle.tcsl_decode(off, t.words.cpu().numpy().view(np.uint32), 1024, 1024),
                          W.view(np.uint16))
