"""The dense/sparse choice per MatMul (Flash-LLM review, section 5 item 5: the
integration's GEMM wrapper picks dense or sparse per weight; section 6, "N
dimension": sparse wins only for skinny N), computed on the host from time
models fitted to B200 measurements of this library's SpMM and of dense cuBLAS
GEMMs.  No device needed."""
import pytest

from unstructured_sparse_skinny_b200 import binding
from unstructured_sparse_skinny_b200.build import build_library


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_library()
    binding.load_library()


# Calls measured on B200 with bench.py (per-call medians, inputs in HBM, CUDA
# graphs): (M, K, N, nnz, sparse us, dense cuBLAS us).  Only cells whose faster
# path is clear (more than 10 % apart) are listed.
MEASURED = [
    (12288, 12288, 8, 75500558, 97.82, 47.32),      # 12288^2, 50 % uniform
    (12288, 12288, 64, 45307139, 100.29, 53.45),    # 12288^2, 70 % uniform
    (12288, 12288, 128, 30202165, 96.26, 51.4),     # 12288^2, 80 % uniform
    (12288, 12288, 128, 7548170, 92.06, 51.4),      # 12288^2, 95 % uniform
    (49152, 12288, 8, 120815616, 169.98, 194.87),   # OPT-175B MLP1, 80 % row magnitude
    (49152, 12288, 16, 60407808, 159.74, 195.28),   # OPT-175B MLP1, 90 % row magnitude
    (36864, 12288, 8, 45305856, 122.88, 141.52),    # OPT-175B QKV, 90 % row magnitude
    (12288, 49152, 16, 60395520, 159.71, 190.26),   # OPT-175B MLP2, 90 % row magnitude
    (36864, 12288, 32, 135880704, 211.17, 141.74),  # OPT-175B QKV, 70 % row magnitude
]


@pytest.mark.parametrize("M,K,N,nnz,t_sparse,t_dense", MEASURED)
def test_matches_clear_measurements(M, K, N, nnz, t_sparse, t_dense):
    assert binding.prefer_sparse(M, K, N, nnz) == (t_sparse < t_dense)
    ps, pd = binding.predict_us(M, K, N, nnz)
    assert abs(ps - t_sparse) / t_sparse < 0.35 and abs(pd - t_dense) / t_dense < 0.15


@pytest.mark.parametrize("M,K", [(12288, 12288), (49152, 12288), (9216, 36864), (4096, 11008)])
def test_monotone_in_sparsity_and_n(M, K):
    # more zeros never turns sparse into dense; a wider N never turns dense into sparse
    for N in (8, 16, 32, 64, 128, 256):
        prev = False
        for s_pct in range(0, 100, 5):
            cur = binding.prefer_sparse(M, K, N, int(M * K * (100 - s_pct) / 100))
            assert cur or not prev
            prev = cur
    for s_pct in (50, 70, 80, 90, 95, 99):
        nnz = int(M * K * (100 - s_pct) / 100)
        prev = True
        for N in (8, 16, 32, 64, 128, 256):
            cur = binding.prefer_sparse(M, K, N, nnz)
            assert prev or not cur
            prev = cur


def test_half_dense_weights_go_dense():
    # at 50 % zeros the format's 4 bytes per entry equal dense fp16's bytes: never sparse
    for M, K in [(12288, 4096), (4096, 4096), (49152, 12288)]:
        for N in (8, 16, 128):
            assert not binding.prefer_sparse(M, K, N, M * K // 2)


def test_bad_arguments():
    lib = binding.load_library()
    assert lib.flashspmm_prefer_sparse(0, 64, 8, 0, 148) == -1
    assert lib.flashspmm_prefer_sparse(64, 64, 300, 0, 148) == -1
    assert lib.flashspmm_prefer_sparse(64, 64, 8, -1, 148) == -1
    assert lib.flashspmm_predict_us(64, 64, 8, 0, 0, None, None) == -1
