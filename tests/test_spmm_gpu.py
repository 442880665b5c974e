"""LSCD SpMM on the GPU vs the fp64 oracle (Flash-LLM review, section 3,
"core formulas": C = A x B; section 5: fp16 inputs, fp32 accumulation).

Bar: every element satisfies |C - C64| <= 2^-10 |C64| + 1e-4 * sum_k |A_mk B_kn|
(fp16 output rounding uses at most 2^-11 |C|; fp32 accumulation over K <= 49152
stays far below the absolute term), and the cases whose exact result is a single
fp16-rounded product are bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import synth
import unstructured_sparse_skinny_b200 as fs
from tests.helpers import assert_parity, gpu_encode, gpu_spmm

pytestmark = pytest.mark.gpu


def _case(M, K, N, s_pct, structure="uniform", key=(200, 0)):
    W = synth.sparse_weight(M, K, s_pct, structure, key)
    B = synth.activations_fp16(N, K, key)
    return W, B


def _oracle(W, B):
    off, words, _ = oracle.tcsl_encode(W)
    C64, absC, _ = oracle.spmm(off, words, W.shape[0], W.shape[1], B, nthreads=8)
    return C64, absC


@pytest.mark.parametrize("split_k", [0, 1, 2, 3, 16])
def test_single_1024_n8(split_k):
    """The single-SpMM workload: 1024 x 1024, 80 % uniform, N = 8, 64 x 64 tiles."""
    W, B = _case(1024, 1024, 8, 80)
    C = gpu_spmm(gpu_encode(W), B, split_k)
    assert_parity(C, *_oracle(W, B), f"split_k={split_k}")


@pytest.mark.parametrize("N", [1, 8, 15, 16, 24, 32, 40, 64, 100, 128, 200, 256])
def test_every_n_bucket(N):
    W, B = _case(1024, 768, N, 80, key=(201, N))
    assert_parity(gpu_spmm(gpu_encode(W), B), *_oracle(W, B), f"N={N}")


@pytest.mark.parametrize("M,K,N", [(200, 136, 9), (64, 64, 16), (192, 520, 16), (1, 8, 1), (4096, 256, 32),
                                   (256, 8192, 16), (130, 72, 8), (320, 1000, 33), (6000, 64, 8)])
@pytest.mark.parametrize("split_k", [0, 2])
def test_ragged_shapes(M, K, N, split_k):
    W, B = _case(M, K, N, 70, key=(202, M))
    assert_parity(gpu_spmm(gpu_encode(W), B, split_k), *_oracle(W, B), f"{M}x{K}x{N}")


@pytest.mark.parametrize("s_pct", [0, 50, 90, 95, 99])
def test_sparsity_range(s_pct):
    W, B = _case(1536, 1024, 32, s_pct, key=(203, s_pct))
    assert_parity(gpu_spmm(gpu_encode(W), B), *_oracle(W, B), f"s={s_pct}")


@pytest.mark.parametrize("structure", ["row_magnitude", "power_law", "column_clustered"])
def test_mask_structures(structure):
    W, B = _case(2048, 2048, 16, 80, structure, key=(204, 0))
    assert_parity(gpu_spmm(gpu_encode(W), B), *_oracle(W, B), structure)


def test_fully_sparse_is_zero():
    W = np.zeros((512, 1024), dtype=np.float16)
    B = synth.activations_fp16(16, 1024, (205, 0))
    C = gpu_spmm(gpu_encode(W), B)
    assert (C.view(np.uint16) & 0x7FFF == 0).all()


@pytest.mark.parametrize("split_k", [0, 1, 4])
def test_permutation_bit_exact(split_k):
    """One nonzero per row: C = fp16_rne(a * b) exactly, whatever the split."""
    g = np.random.default_rng(17)
    M = K = 1024
    perm = g.permutation(K)
    a = (g.standard_normal(M) * 0.5).astype(np.float16)
    a[a == 0] = 1
    W = np.zeros((M, K), dtype=np.float16)
    W[np.arange(M), perm] = a
    B = synth.activations_fp16(24, K, (206, 0))
    C = gpu_spmm(gpu_encode(W), B, split_k)
    exact = (a.astype(np.float64)[None, :] * B.astype(np.float64)[:, perm]).astype(np.float16)
    assert C.view(np.uint16).tobytes() == exact.view(np.uint16).tobytes()


def test_dense_matches_torch_matmul():
    """0 % sparsity: also compare with torch's dense fp16 GEMM (fp32 accumulate)."""
    W, B = _case(1024, 2048, 64, 0, key=(207, 0))
    C = gpu_spmm(gpu_encode(W), B)
    ref = (torch.from_numpy(B).cuda().float() @ torch.from_numpy(W).cuda().float().t()).cpu().numpy()
    assert np.allclose(C.astype(np.float32), ref, rtol=2e-3, atol=2e-3)
    assert_parity(C, *_oracle(W, B), "dense")


def test_overflow_to_inf_and_exact_max():
    W = np.zeros((128, 64), dtype=np.float16)
    W[0, 0] = 65504.0
    W[1, 0] = 60000.0
    W[1, 1] = 60000.0
    B = np.zeros((16, 64), dtype=np.float16)
    B[:, 0] = 1.0
    B[:, 1] = 1.0
    C = gpu_spmm(gpu_encode(W), B)
    assert (C[:, 0] == np.float16(65504.0)).all()
    assert np.isinf(C[:, 1]).all() and (C[:, 1] > 0).all()


def test_deterministic_for_fixed_split():
    W, B = _case(4096, 4096, 16, 80, key=(208, 0))
    t = gpu_encode(W)
    for split_k in (0, 3):
        c1 = gpu_spmm(t, B, split_k)
        c2 = gpu_spmm(t, B, split_k)
        assert c1.tobytes() == c2.tobytes()


def test_k_zero_and_empty_outputs():
    W = np.zeros((128, 0), dtype=np.float16)
    t = gpu_encode(W)
    C = fs.spmm_lscd(t, torch.empty((8, 0), dtype=torch.float16, device="cuda"),
                     C=torch.full((8, 128), 7.0, dtype=torch.float16, device="cuda"))
    assert (C == 0).all()
    t = gpu_encode(np.zeros((0, 64), dtype=np.float16))
    C = fs.spmm_lscd(t, torch.zeros((8, 64), dtype=torch.float16, device="cuda"))
    assert C.shape == (8, 0)


def test_host_buffer_entry_point_matches_device_path():
    W, B = _case(2048, 1024, 32, 80, key=(209, 0))
    t = gpu_encode(W)
    dev = gpu_spmm(t, B)
    B_host = torch.from_numpy(B).pin_memory()
    C_host = torch.empty((32, 2048), dtype=torch.float16).pin_memory()
    B_dev = torch.empty((32, 1024), dtype=torch.float16, device="cuda")
    C_dev = torch.empty((32, 2048), dtype=torch.float16, device="cuda")
    fs.spmm_lscd_host(t, B_host, C_host, B_dev, C_dev)
    torch.cuda.synchronize()
    fs.check_device_status()
    assert C_host.numpy().tobytes() == dev.tobytes()


def test_corrupt_data_is_contained_and_reported():
    """A word with an out-of-tile loc is skipped by the SpMM (memory-safe, result
    unspecified) and reported by the validator; corrupt tile offsets are
    reported by the SpMM itself."""
    W, B = _case(512, 512, 8, 80, key=(210, 0))
    t = gpu_encode(W)
    w = t.words.clone()
    w[1] = int(np.uint32(0x3C00 | (5000 << 16)).view(np.int32))  # loc beyond the tile
    bad = fs.TCSL(t.tile_offsets, w, t.nnz, t.M, t.K)
    fs.spmm_lscd(bad, torch.from_numpy(B).cuda())
    fs.check_device_status()  # the SpMM does not check word contents
    with pytest.raises(fs.FlashSpmmError) as e:
        fs.tcsl_validate(bad)
    assert e.value.status == 6
    off = t.tile_offsets.clone()
    off[1] += 1  # misaligned tile start: the tile is skipped and flagged
    bad = fs.TCSL(off, t.words, t.nnz, t.M, t.K)
    fs.spmm_lscd(bad, torch.from_numpy(B).cuda())
    with pytest.raises(fs.FlashSpmmError) as e:
        fs.check_device_status()
    assert e.value.status == 6
    fs.check_device_status()  # cleared


def test_workspace_too_small_is_rejected():
    W, B = _case(4096, 4096, 16, 80, key=(211, 0))
    t = gpu_encode(W)
    need = fs.spmm_workspace_bytes(4096, 4096, 16, 0)
    assert need > 0
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(fs.FlashSpmmError) as e:
        fs.spmm_lscd(t, torch.from_numpy(B).cuda(), workspace=ws)
    assert e.value.status == 4


@pytest.mark.parametrize("s_pct", [95, 99])
def test_many_short_tiles_high_sparsity(s_pct):
    """Large, very sparse problem: every strip tile is one short load round
    (the 16-word-round instance), so the decompress warps turn over their two
    buffer sets far more often than they expand words and the MMA warp issues
    many groups per unit (a liveness case: must finish without a timeout,
    within the bound)."""
    W, B = _case(9216, 9216, 8, s_pct, key=(212, s_pct))
    assert_parity(gpu_spmm(gpu_encode(W), B), *_oracle(W, B), f"9216^2 s={s_pct}")


@pytest.mark.parametrize("N", [8, 64])
def test_sparse_matrix_with_dense_tiles(N):
    """A very sparse matrix holding one fully dense 64 x 64 tile (4096 words:
    sixteen full batches for one warp) and one dense row segment."""
    W, B = _case(1024, 1024, N, 95, key=(213, N))
    g = np.random.default_rng(213)
    W[128:192, 320:384] = (g.standard_normal((64, 64)) * 0.02).astype(np.float16)
    W[600, 0:512] = (g.standard_normal(512) * 0.02).astype(np.float16)
    assert_parity(gpu_spmm(gpu_encode(W), B), *_oracle(W, B), f"dense tiles N={N}")


@pytest.mark.parametrize("r0,r1", [(0, 640), (640, 1000), (192, 448), (960, 1000)])
def test_row_slice_shard(r0, r1):
    """A row-split shard (a view sharing the full matrix's words) multiplies to
    the same rows of the product."""
    W, B = _case(1000, 768, 16, 80, key=(214, 0))
    t = gpu_encode(W)
    shard = t.slice_rows(r0, r1)
    C = fs.spmm_lscd(shard, torch.from_numpy(B).cuda())
    fs.check_device_status()
    off, words, _ = oracle.tcsl_encode(W)
    C64, absC = oracle.spmm_rows(off, words, 1000, 768, B, np.arange(r0, r1))
    assert_parity(C.cpu().numpy().T, C64, absC, f"rows {r0}:{r1}")


@pytest.mark.parametrize("structure,s_pct,N", [("uniform", 80, 8), ("uniform", 70, 32), ("power_law", 90, 16),
                                               ("column_clustered", 80, 64), ("row_magnitude", 50, 128),
                                               ("uniform", 95, 256)])
def test_bank_balanced_word_order(structure, s_pct, N):
    """The SpMM reads either word order: bank-balanced (v2) words give a product
    within the same bound (the scatter does not depend on the order)."""
    W, B = _case(2048, 1536, N, s_pct, structure, key=(210, s_pct))
    t = fs.tcsl_encode(torch.from_numpy(W).cuda(), order=1)
    fs.check_device_status()
    assert_parity(gpu_spmm(t, B), *_oracle(W, B), f"v2 {structure} {s_pct}% N={N}")


def test_workspace_counters_left_zero_across_plans():
    """One workspace, zeroed once, serves calls with different plans: every
    completed call leaves its arrival counters zero, and the partial sums of
    one call never land where a later call keeps its counters."""
    ws = torch.zeros(1 << 24, dtype=torch.uint8, device="cuda")
    for M, K, N in [(4096, 4096, 32), (1024, 2048, 8), (9216, 1024, 64), (4096, 4096, 32)]:
        W, B = _case(M, K, N, 80, key=(215, M + N))
        need = fs.spmm_workspace_bytes(M, K, N, 0)
        assert 4096 < need <= ws.numel()  # these shapes share units between pieces
        C = fs.spmm_lscd(gpu_encode(W), torch.from_numpy(B).cuda(), workspace=ws)
        fs.check_device_status()
        assert_parity(C.cpu().numpy(), *_oracle(W, B), f"{M}x{K}x{N}")
        assert int(ws[:4096].count_nonzero()) == 0
