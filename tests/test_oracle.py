"""Pins for the CPU oracle (no GPU needed).

Each pin checks the oracle against something other than itself: hand-derived
golden words and products, the brute-force dense product, closed forms,
numpy's own IEEE fp16 conversions, invariants of the format definition
(Flash-LLM paper review, section 3, "sparse encoding format: Tiled-CSL") and
the compute-intensity numbers printed on the same page (section 3, "core
formulas": tensor-core use of 5.1/10.3/20.5/40.1 % at N = 8/16/32/64 for
M = 48K, K = 12K).
"""
import json
from pathlib import Path

import numpy as np
import pytest

import oracle
import synth

GOLDEN = json.loads((Path(__file__).parent / "golden" / "tcsl_worked_examples.json").read_text())


def _dense_from_nonzeros(ex):
    A = np.zeros((ex["M"], ex["K"]), dtype=np.uint16)
    for r, c, h in ex["nonzeros"]:
        A[r, c] = int(h, 16)
    return A


@pytest.mark.parametrize("ex", GOLDEN["examples"], ids=lambda e: e["name"])
def test_golden_encode(ex):
    A = _dense_from_nonzeros(ex)
    off, words, nnz = oracle.tcsl_encode(A, ex["tile_m"], ex["tile_k"])
    assert off.tolist() == ex["tile_offsets"]
    assert [f"{w:08X}" for w in words] == ex["words"]
    assert nnz == ex["nnz"]


@pytest.mark.parametrize("ex", GOLDEN["examples"], ids=lambda e: e["name"])
def test_golden_decode(ex):
    off = np.array(ex["tile_offsets"], dtype=np.int32)
    words = np.array([int(w, 16) for w in ex["words"]], dtype=np.uint32)
    A = oracle.tcsl_decode(off, words, ex["M"], ex["K"], ex["tile_m"], ex["tile_k"])
    assert np.array_equal(A, _dense_from_nonzeros(ex))


def test_golden_spmm():
    ex = GOLDEN["examples"][0]
    off = np.array(ex["tile_offsets"], dtype=np.int32)
    words = np.array([int(w, 16) for w in ex["words"]], dtype=np.uint32)
    B = np.array(ex["B_NK"], dtype=np.float16)
    C64, absC, C16 = oracle.spmm(off, words, ex["M"], ex["K"], B, ex["tile_m"], ex["tile_k"])
    expect = np.array(ex["C_NM"], dtype=np.float64)
    assert np.array_equal(C64, expect)
    assert np.array_equal(C16.astype(np.float64), expect)
    # sum |a b| for row 0, n = 0: |1*2| + |-0*4| + |2*5| = 12
    assert absC[0, 0] == 12.0


# ---------------------------------------------------------------- round trip

def _random_matrix(M, K, density, seed, specials=False):
    g = np.random.default_rng(seed)
    A = (g.standard_normal((M, K)) * 0.02).astype(np.float16)
    A[g.random((M, K)) >= density] = 0
    bits = A.view(np.uint16)
    if specials:
        pick = g.random((M, K))
        bits[pick < 0.01] = 0x8000  # -0.0
        bits[(pick >= 0.01) & (pick < 0.015)] = 0x7E00  # NaN
        bits[(pick >= 0.015) & (pick < 0.02)] = 0xFC00  # -Inf
        bits[(pick >= 0.02) & (pick < 0.03)] = 0x0001  # smallest subnormal
    return bits


SHAPES = [  # (M, K, tile_m, tile_k)
    (128, 128, 64, 64), (200, 136, 64, 64), (64, 64, 64, 64), (1, 1, 64, 64),
    (130, 70, 128, 64), (37, 29, 16, 8), (9, 11, 2, 4), (5, 7, 1, 1), (300, 300, 255, 257),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("density", [0.0, 0.05, 0.2, 0.5, 1.0])
def test_round_trip_and_invariants(shape, density):
    M, K, tm, tk = shape
    A = _random_matrix(M, K, density, seed=M * 1000 + K, specials=True)
    off, words, nnz = oracle.tcsl_encode(A, tm, tk)
    # decode(encode(A)) == A, bit for bit (keeps -0.0, NaN payloads, Inf, subnormals)
    assert np.array_equal(oracle.tcsl_decode(off, words, M, K, tm, tk), A)
    _check_invariants(A, off, words, nnz, tm, tk)


def _check_invariants(A, off, words, nnz, tm, tk):
    M, K = A.shape
    TM, TK = -(-M // tm), -(-K // tk)
    assert off.size == TM * TK + 1 and off[0] == 0
    assert off[-1] == words.size
    seg = np.diff(off)
    assert (seg >= 0).all() and (seg % 4 == 0).all()
    assert nnz == int(np.count_nonzero(A))
    total_real = 0
    for t in range(TM * TK):
        w = words[off[t]:off[t + 1]]
        loc = w >> 16
        real = loc != 0xFFFF
        n_real = int(real.sum())
        total_real += n_real
        # sentinels only after the last real word, and exactly 0xFFFF0000
        assert real[:n_real].all() and not real[n_real:].any()
        assert (w[n_real:] == oracle.SENTINEL).all()
        assert w.size - n_real < 4
        # locs strictly ascending, inside the tile, value bits never zero
        locs = loc[:n_real].astype(np.int64)
        assert (np.diff(locs) > 0).all()
        assert (locs < tm * tk).all()
        assert ((w[:n_real] & 0xFFFF) != 0).all()
        i, j = divmod(t, TK)
        r, c = locs // tk, locs % tk
        assert (i * tm + r < M).all() and (j * tk + c < K).all()
    assert total_real == nnz


def test_empty_and_full_tiles():
    A = np.zeros((128, 128), dtype=np.uint16)
    A[:64, :64] = 0x3C00  # tile 0 fully dense: 4096 words, no padding
    off, words, nnz = oracle.tcsl_encode(A)
    assert off.tolist() == [0, 4096, 4096, 4096, 4096]
    assert nnz == 4096
    assert ((words >> 16) == np.arange(4096)).all()
    A0 = np.zeros((128, 192), dtype=np.uint16)
    off0, words0, nnz0 = oracle.tcsl_encode(A0)
    assert off0.tolist() == [0] * 7 and words0.size == 0 and nnz0 == 0


def test_single_nonzero_first_and_last_loc():
    for loc in (0, 4095):
        A = np.zeros((64, 64), dtype=np.uint16)
        A[loc // 64, loc % 64] = 0x1234
        off, words, _ = oracle.tcsl_encode(A)
        assert off.tolist() == [0, 4]
        assert words.tolist() == [0x1234 | (loc << 16)] + [oracle.SENTINEL] * 3


def test_tile_area_limit():
    A = np.zeros((256, 256), dtype=np.uint16)
    with pytest.raises(oracle.OracleError):
        oracle.tcsl_encode(A, 256, 256)  # 65536 locations would collide with the sentinel


def test_decode_rejects_out_of_tile_loc():
    off = np.array([0, 4], dtype=np.int32)
    words = np.array([0x3C00 | (4096 << 16)] + [oracle.SENTINEL] * 3, dtype=np.uint32)
    with pytest.raises(oracle.OracleError):
        oracle.tcsl_decode(off, words, 64, 64)


# ---------------------------------------------------------------- SpMM pins

@pytest.mark.parametrize("M,K,N,tm,tk,density", [
    (64, 64, 8, 64, 64, 0.2), (130, 200, 16, 64, 64, 0.3), (96, 256, 5, 32, 64, 0.1),
    (17, 33, 3, 4, 8, 0.5), (256, 128, 9, 64, 64, 1.0), (64, 128, 1, 64, 64, 0.05)])
def test_spmm_equals_dense_bruteforce(M, K, N, tm, tk, density):
    """Sparse-list sum == dense triple loop bit for bit (up to the sign of zero):
    both add the same exact fp64 products in ascending k, and an exact +-0
    product cannot change a nonzero sum."""
    A = _random_matrix(M, K, density, seed=7 + M + K)
    g = np.random.default_rng(N)
    B = g.standard_normal((N, K)).astype(np.float16)
    off, words, _ = oracle.tcsl_encode(A, tm, tk)
    C64, absC, C16 = oracle.spmm(off, words, M, K, B, tm, tk)
    D = oracle.dense(A, B)
    assert np.array_equal(C64 == 0, D == 0)
    nz = C64 != 0
    assert np.array_equal(C64[nz], D[nz])
    # absC bounds |C| and equals the dense sum of |a b|
    absD = oracle.dense(np.abs(A.view(np.float16)), np.abs(B))
    assert np.array_equal(absC, absD)
    assert (np.abs(C64) <= absC).all()
    # C16 is the fp16 RNE rounding of C64 (numpy converts float64 -> float16 directly)
    assert np.array_equal(C16.view(np.uint16), C64.astype(np.float16).view(np.uint16))


def test_spmm_threads_bit_identical():
    A = _random_matrix(640, 320, 0.25, seed=3)
    B = np.random.default_rng(1).standard_normal((12, 320)).astype(np.float16)
    off, words, _ = oracle.tcsl_encode(A)
    one = oracle.spmm(off, words, 640, 320, B, nthreads=1)
    many = oracle.spmm(off, words, 640, 320, B, nthreads=7)
    for a, b in zip(one, many):
        assert np.array_equal(a.view(np.uint8), b.view(np.uint8))


def test_spmm_rows_matches_full():
    A = _random_matrix(200, 136, 0.3, seed=5)
    B = np.random.default_rng(2).standard_normal((6, 136)).astype(np.float16)
    off, words, _ = oracle.tcsl_encode(A)
    C64, absC, _ = oracle.spmm(off, words, 200, 136, B)
    rows = np.array([199, 0, 64, 63, 128, 7])
    R64, Rabs = oracle.spmm_rows(off, words, 200, 136, B, rows)
    assert np.array_equal(R64, C64[:, rows].T)
    assert np.array_equal(Rabs, absC[:, rows].T)


def test_fully_sparse_gives_zero():
    A = np.zeros((192, 256), dtype=np.uint16)
    B = np.random.default_rng(0).standard_normal((16, 256)).astype(np.float16)
    off, words, _ = oracle.tcsl_encode(A)
    C64, absC, C16 = oracle.spmm(off, words, 192, 256, B)
    assert (C64 == 0).all() and (absC == 0).all() and (C16 == 0).all()


def test_permutation_is_exact_product():
    """One nonzero per row: C = fp16(a * b) exactly (the fp16 product is exact in fp64)."""
    g = np.random.default_rng(11)
    M = K = 256
    perm = g.permutation(K)
    a = (g.standard_normal(M) * 0.5).astype(np.float16)
    a[a == 0] = np.float16(1.0)
    A = np.zeros((M, K), dtype=np.float16)
    A[np.arange(M), perm] = a
    B = g.standard_normal((8, K)).astype(np.float16)
    off, words, _ = oracle.tcsl_encode(A)
    C64, _, C16 = oracle.spmm(off, words, M, K, B)
    exact = a.astype(np.float64)[None, :] * B.astype(np.float64)[:, perm]
    assert np.array_equal(C64, exact)
    assert np.array_equal(C16.view(np.uint16), exact.astype(np.float16).view(np.uint16))


def test_closed_form_ones():
    """A = mask of ones with n_r ones in row r, B = ones: C[n, r] = n_r exactly."""
    g = np.random.default_rng(4)
    M, K = 128, 448
    mask = g.random((M, K)) < 0.3
    A = mask.astype(np.float16)
    B = np.ones((4, K), dtype=np.float16)
    off, words, _ = oracle.tcsl_encode(A)
    C64, absC, C16 = oracle.spmm(off, words, M, K, B)
    assert np.array_equal(C64, np.broadcast_to(mask.sum(1).astype(np.float64), (4, M)))
    assert np.array_equal(absC, C64)


def test_closed_form_arithmetic_series():
    """Dense row of ones times B[k, n] = (k + 1) * 2^-n gives (K(K+1)/2) * 2^-n."""
    M, K = 64, 320
    A = np.ones((M, K), dtype=np.float16)
    B = np.stack([(np.arange(K) + 1) * 2.0 ** -n for n in range(3)]).astype(np.float16)
    off, words, nnz = oracle.tcsl_encode(A)
    assert nnz == M * K and words.size == M * K  # dense tiles carry no padding
    C64, _, _ = oracle.spmm(off, words, M, K, B)
    for n in range(3):
        assert (C64[n] == K * (K + 1) / 2 * 2.0 ** -n).all()


def test_fp16_output_overflow_rounds_to_inf():
    A = np.zeros((64, 64), dtype=np.float16)
    A[0, 0] = 60000.0
    A[0, 1] = 60000.0
    A[1, 0] = 65504.0
    B = np.zeros((1, 64), dtype=np.float16)
    B[0, 0] = 1.0
    B[0, 1] = 0.0917  # 60000 * (1 + 0.0917...) ~ 65500: rounds to a finite value or Inf by RNE
    off, words, _ = oracle.tcsl_encode(A)
    C64, _, C16 = oracle.spmm(off, words, 64, 64, B)
    assert np.array_equal(C16.view(np.uint16), C64.astype(np.float16).view(np.uint16))
    assert C16[0, 1] == np.float16(65504.0)


# ---------------------------------------------------------------- conversions

def test_half_to_double_all_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.half_to_double(h)
    ref = h.view(np.float16).astype(np.float64)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_double_to_half_matches_numpy():
    g = np.random.default_rng(9)
    x = np.concatenate([
        g.standard_normal(200000) * 10.0 ** g.integers(-9, 6, 200000),
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 1e9, -1e9, np.inf, -np.inf,
                  2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 3 * 2.0 ** -26, 2.0 ** -14,
                  2.0 ** -14 - 2.0 ** -25, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2049.0, 2051.0]),
        # exact midpoints between adjacent fp16 values: ties must go to even
        (np.arange(1, 65504, 97, dtype=np.float64) + 0.5),
    ])
    ours = oracle.double_to_half(x)
    ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)
    assert oracle.double_to_half(np.array([np.nan]))[0] & 0x7E00 == 0x7E00


# ---------------------------------------------------------------- compute intensity

def test_ci_bound_and_limit():
    for M, K, N in [(1024, 1024, 8), (49152, 12288, 64), (16, 16, 16), (12288, 4096, 128)]:
        assert oracle.ci(M, K, N) <= N
    assert abs(oracle.ci(1e12, 1e12, 16) - 16) < 1e-6
    # symmetric in M and K
    assert oracle.ci(300, 700, 8) == oracle.ci(700, 300, 8)


def test_ci_reproduces_printed_tensor_core_use():
    """The page prints 5.1/10.3/20.5/40.1 % tensor-core use for M=48K, K=12K at
    N = 8/16/32/64 with HBM saturated; use is CI x (BW / peak), so the ratios to
    N = 8 must follow CI's ratios without any hardware constant."""
    printed = {8: 5.1, 16: 10.3, 32: 20.5, 64: 40.1}
    base = oracle.ci(48 * 1024, 12 * 1024, 8)
    for n, pct in printed.items():
        ratio = oracle.ci(48 * 1024, 12 * 1024, n) / base
        assert abs(ratio - pct / printed[8]) / (pct / printed[8]) < 0.03


def test_tolerance_bound_semantics():
    C64 = np.array([1.0, 0.0, np.nan, np.inf, 2.0])
    absC = np.array([1.0, 5.0, 1.0, 1.0, 2.0])
    ok = oracle.tolerance_ok(np.array([1.0 + 2 ** -11, 4e-4, np.nan, np.inf, 2.1]), C64, absC)
    assert ok.tolist() == [True, True, True, True, False]


# ---------------------------------------------------------------- generators

def test_generators_reproducible_and_shaped():
    W1 = synth.sparse_weight(256, 320, 80, "uniform", (9, 0))
    W2 = synth.sparse_weight(256, 320, 80, "uniform", (9, 0))
    assert W1.dtype == np.float16 and W1.shape == (256, 320)
    assert np.array_equal(W1.view(np.uint16), W2.view(np.uint16))
    assert abs(np.mean(W1 == 0) - 0.8) < 0.01
    nz = W1[W1 != 0].astype(np.float64)
    assert abs(nz.std() - 0.02) < 0.002


def test_row_magnitude_exact_counts():
    for s in (50, 70, 90):
        W = synth.sparse_weight(64, 1000, s, "row_magnitude", (9, 1))
        drop = synth.row_magnitude_drop_count(1000, s)
        assert ((W == 0).sum(1) == drop).all()
        full = synth.weights_fp16(64, 1000, (9, 1, s, synth.STRUCTURES["row_magnitude"]))
        kept = np.abs(full.astype(np.float32)) * (W != 0)
        lost = np.abs(full.astype(np.float32)) * (W == 0)
        assert (lost.max(1) <= np.where(W != 0, kept, np.inf).min(1)).all()


def test_power_law_and_clustered_densities():
    for s in (0.5, 0.7, 0.9, 0.95):
        alpha = synth.power_law_alpha(1 - s)
        d = synth.power_law_sample(np.random.default_rng(0).random(400000), alpha)
        assert abs(d.mean() - (1 - s)) < 0.003
        assert d.min() >= 0.02 - 1e-12 and d.max() <= 0.60 + 1e-12
    W = synth.sparse_weight(512, 1024, 80, "power_law", (9, 2))
    assert abs(np.mean(W != 0) - 0.2) < 0.03
    W = synth.sparse_weight(512, 1024, 80, "column_clustered", (9, 3))
    dens_blocks = (W != 0).reshape(512, 16, 64).mean(axis=(0, 2))
    d_h, d_c = synth.column_cluster_densities(0.8)
    hot = dens_blocks > (d_h + d_c) / 2
    assert hot.sum() == 4
    assert abs(dens_blocks[hot].mean() - d_h) < 0.01 and abs(dens_blocks[~hot].mean() - d_c) < 0.01
