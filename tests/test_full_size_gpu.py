"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (automatic split, one CTA per SM).

For every matrix: the GPU Tiled-CSL encoding is compared byte for byte with
the oracle's encoding of the same seeded matrix, and the product is checked on
a sample of output rows (tile edges plus seeded random rows, all N columns)
that the oracle computes one by one, with the same element-wise bound as the
small parity tests.  Shapes: the OPT-66B and OPT-175B decoder layers of the
Flash-LLM review's kernel benchmark (section 6), a LLaMA-7B-shaped 50 % layer
and cells of the 12288^2 stress sweep, including the largest M (49152) and
the largest K (49152)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import unstructured_sparse_skinny_b200 as fs

pytestmark = pytest.mark.gpu

# (config, layer index, name, M, K, sparsity %, structure, Ns)
CASES = [
    (2, 0, "opt66b_qkv", 27648, 9216, 80, "uniform", (8, 16, 32, 64)),
    (2, 1, "opt66b_out_proj", 9216, 9216, 80, "uniform", (8, 16, 32, 64)),
    (2, 2, "opt66b_mlp1", 36864, 9216, 80, "uniform", (8, 16, 32, 64)),
    (2, 3, "opt66b_mlp2", 9216, 36864, 80, "uniform", (8, 16, 32, 64)),
    (3, 1, "opt175b_out_proj_70", 12288, 12288, 70, "row_magnitude", (8, 16, 32)),
    (3, 1, "opt175b_out_proj_80", 12288, 12288, 80, "row_magnitude", (8, 16, 32)),
    (3, 1, "opt175b_out_proj_90", 12288, 12288, 90, "row_magnitude", (8, 16, 32)),
    (3, 2, "opt175b_mlp1_90", 49152, 12288, 90, "row_magnitude", (32,)),
    (3, 3, "opt175b_mlp2_70", 12288, 49152, 70, "row_magnitude", (8,)),
    (4, 0, "llama7b_qkv", 12288, 4096, 50, "row_magnitude", (8, 64, 128)),
    (4, 4, "llama7b_down", 4096, 11008, 50, "row_magnitude", (8, 128)),
    (5, 0, "stress_95_clustered", 12288, 12288, 95, "column_clustered", (128,)),
    (5, 0, "stress_50_powerlaw", 12288, 12288, 50, "power_law", (8,)),
    (5, 0, "stress_60_uniform", 12288, 12288, 60, "uniform", (64,)),
]


def _sample_rows(M, seed, count=96):
    g = np.random.default_rng(seed)
    edges = [0, 1, 63, 64, 127, 128, M // 2, M - 65, M - 64, M - 1]
    return np.unique(np.concatenate([np.array(edges), g.integers(0, M, count)]))


@pytest.mark.parametrize("case", CASES, ids=[c[2] for c in CASES])
def test_full_size(case):
    cfg, layer, name, M, K, s_pct, structure, Ns = case
    key = synth.layer_key(cfg, layer)
    W = synth.sparse_weight(M, K, s_pct, structure, key)
    t = fs.tcsl_encode(torch.from_numpy(W).cuda())
    fs.check_device_status()
    off, words, nnz = oracle.tcsl_encode(W)
    del W
    assert t.nnz == nnz
    assert np.array_equal(t.tile_offsets.cpu().numpy(), off)
    assert t.words.cpu().numpy().view(np.uint32).tobytes() == words.tobytes()
    rows = _sample_rows(M, M + K + s_pct)
    for N in Ns:
        B = synth.activations_fp16(N, K, key)
        C = fs.spmm_lscd(t, torch.from_numpy(B).cuda())
        fs.check_device_status()
        got = C[:, torch.from_numpy(rows).cuda()].cpu().numpy().T  # [rows, N]
        C64, absC = oracle.spmm_rows(off, words, M, K, B, rows)
        ok = oracle.tolerance_ok(got, C64, absC)
        assert ok.all(), (f"{name} N={N}: {int((~ok).sum())} of {ok.size} sampled elements outside the bound; "
                          f"first at row {rows[np.argwhere(~ok)[0][0]]}")
