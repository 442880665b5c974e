"""Word-balanced piece tables, K-range views and fp32 output on the GPU.

* The device partition kernel writes the same table as the host rule
  (flashspmm_partition_host, checked against a restatement on the CPU).
* The SpMM run on a table's pieces meets the oracle bound on every mask
  structure; a malformed table is reported (CORRUPT_FORMAT) and the SpMM
  falls back to even pieces, still correct; a table made for another SM count
  is ignored.
* K-range views (tensor-parallel K split: the Flash-LLM review, section 5
  item 5, distributed inference) multiply to the oracle's product of the same
  columns, in fp32; the fp32 partials of a K split sum to the full product.
* fp32 output holds the accumulators the fp16 output rounds: the two agree bit
  for bit after round-to-nearest-even."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import synth
import unstructured_sparse_skinny_b200 as fs
from tests.helpers import assert_parity

pytestmark = pytest.mark.gpu


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _encode(W, partition=False):
    t = fs.tcsl_encode(torch.from_numpy(np.ascontiguousarray(W)).cuda(), partition=partition)
    fs.check_device_status()
    return t


def _oracle(W, B):
    off, words, _ = oracle.tcsl_encode(np.ascontiguousarray(W))
    C64, absC, _ = oracle.spmm(off, words, W.shape[0], W.shape[1], B, nthreads=8)
    return C64, absC


def _run(t, B, dtype=torch.float16, split_k=0):
    N = B.shape[0]
    C = torch.empty((N, t.M), dtype=dtype, device="cuda")
    fs.spmm_lscd(t, torch.from_numpy(np.ascontiguousarray(B)).cuda(), C, split_k=split_k)
    return C


def assert_parity_f32(C32, C64, absC, what=""):
    """fp32 output: the accumulation term of the bound, no output rounding."""
    err = np.abs(C32.astype(np.float64) - C64)
    ok = err <= 1e-4 * absC + 2.0 ** -24 * np.abs(C64)
    assert ok.all(), f"{what}: {int((~ok).sum())} of {ok.size} outside; worst {err.max()!r}"


@pytest.mark.parametrize("M,K,structure,s_pct", [(4096, 4096, "power_law", 80), (2048, 3072, "column_clustered", 90),
                                                 (1000, 1000, "row_magnitude", 70), (330, 200, "uniform", 80),
                                                 (6000, 64, "power_law", 60), (12288, 12288, "power_law", 90)])
def test_device_table_matches_host_rule(M, K, structure, s_pct):
    W = synth.sparse_weight(M, K, s_pct, structure, (230, s_pct))
    t = _encode(W, partition=True)
    P = fs.partition_pieces(M, K, _sms())
    assert t.piece_bounds.numel() == P + 1
    host = fs.partition_host(t.tile_offsets.cpu().numpy(), M, K, P)
    assert t.piece_bounds.cpu().tolist() == host


@pytest.mark.parametrize("M,K,N,structure,s_pct", [
    (4096, 4096, 16, "power_law", 80), (4096, 4096, 8, "power_law", 90), (2048, 3072, 32, "column_clustered", 80),
    (1000, 1000, 64, "row_magnitude", 70), (330, 200, 9, "uniform", 80), (6000, 64, 16, "power_law", 60),
    (1024, 1024, 8, "uniform", 80), (640, 8192, 128, "power_law", 70), (128, 128, 256, "uniform", 50)])
def test_spmm_on_table_pieces(M, K, N, structure, s_pct):
    W = synth.sparse_weight(M, K, s_pct, structure, (231, M))
    B = synth.activations_fp16(N, K, (231, N))
    t = _encode(W, partition=True)
    C = _run(t, B)
    fs.check_device_status()
    assert_parity(C.cpu().numpy(), *_oracle(W, B), f"table {M}x{K} {structure} {s_pct}% N={N}")


def test_malformed_table_is_reported_and_ignored():
    W = synth.sparse_weight(2048, 2048, 80, "power_law", (232, 0))
    B = synth.activations_fp16(16, 2048, (232, 0))
    t = _encode(W, partition=True)
    bad = t.piece_bounds.clone()
    bad[3] = bad[2]                        # an empty piece: not strictly increasing
    C = _run(dataclasses.replace(t, piece_bounds=bad), B)
    with pytest.raises(fs.FlashSpmmError) as e:
        fs.check_device_status()
    assert e.value.status == 6             # FLASHSPMM_ERR_CORRUPT_FORMAT
    assert_parity(C.cpu().numpy(), *_oracle(W, B), "even pieces after a malformed table")
    fs.check_device_status()


def test_table_for_another_sm_count_is_ignored():
    W = synth.sparse_weight(2048, 2048, 80, "power_law", (233, 0))
    B = synth.activations_fp16(16, 2048, (233, 0))
    t = _encode(W).partition(num_sms=_sms() // 2)
    assert t.piece_bounds.numel() - 1 != fs.partition_pieces(2048, 2048, _sms())
    C = _run(t, B)
    fs.check_device_status()
    assert_parity(C.cpu().numpy(), *_oracle(W, B), "table of another plan")


def test_fp32_output_rounds_to_the_fp16_output():
    """Same plan, same accumulators: fp16 C == RNE(fp32 C) bit for bit, and the
    fp32 C meets the accumulation bound."""
    for structure, N, split_k in (("uniform", 16, 0), ("power_law", 64, 0), ("column_clustered", 8, 3)):
        W = synth.sparse_weight(1536, 2048, 80, structure, (234, N))
        B = synth.activations_fp16(N, 2048, (234, N))
        t = _encode(W)
        C16 = _run(t, B, split_k=split_k)
        C32 = _run(t, B, torch.float32, split_k=split_k)
        fs.check_device_status()
        assert torch.equal(C32.half().view(torch.int16), C16.view(torch.int16)), structure
        assert_parity_f32(C32.cpu().numpy(), *_oracle(W, B), f"fp32 {structure}")


@pytest.mark.parametrize("M,K,N,k0,k1", [(1536, 2048, 16, 0, 512), (1536, 2048, 16, 512, 2048),
                                         (1536, 2048, 32, 1024, 1088), (1000, 1000, 8, 960, 1000),
                                         (1000, 1000, 64, 64, 704), (300, 4096, 128, 2048, 4096)])
def test_k_range_view(M, K, N, k0, k1):
    """A K-range view of the encoded matrix multiplies to the oracle's product
    of those columns (fp32 output), with and without a piece table."""
    W = synth.sparse_weight(M, K, 80, "power_law", (235, k0))
    B = synth.activations_fp16(N, K, (235, k1))
    t = _encode(W)
    v = t.slice_cols(k0, k1)
    Bs = np.ascontiguousarray(B[:, k0:k1])
    want = _oracle(W[:, k0:k1], Bs)
    for view in (v, v.partition()):
        C32 = _run(view, Bs, torch.float32)
        fs.check_device_status()
        assert_parity_f32(C32.cpu().numpy(), *want, f"K view {k0}:{k1}")


def test_k_split_partials_sum_to_the_product():
    """Tensor-parallel K split on one GPU: each shard's fp32 partial, summed
    (what an all-reduce computes), meets the bound for the full product."""
    M, K, N = 2048, 3072, 16
    W = synth.sparse_weight(M, K, 80, "uniform", (236, 0))
    B = synth.activations_fp16(N, K, (236, 0))
    t = _encode(W)
    total = torch.zeros((N, M), dtype=torch.float32, device="cuda")
    for k0, k1 in ((0, 1024), (1024, 2048), (2048, 3072)):
        total += _run(t.slice_cols(k0, k1), np.ascontiguousarray(B[:, k0:k1]), torch.float32)
    fs.check_device_status()
    assert_parity_f32(total.cpu().numpy(), *_oracle(W, B), "sum of K shards")


def test_row_view_of_k_view():
    """Views compose: rows of a K-range view address the same tiles."""
    M, K, N = 1000, 2048, 16
    W = synth.sparse_weight(M, K, 70, "uniform", (237, 0))
    B = synth.activations_fp16(N, K, (237, 0))
    t = _encode(W)
    v = t.slice_cols(512, 1536).slice_rows(192, 1000)
    Bs = np.ascontiguousarray(B[:, 512:1536])
    C32 = _run(v, Bs, torch.float32)
    fs.check_device_status()
    assert_parity_f32(C32.cpu().numpy(), *_oracle(W[192:1000, 512:1536], Bs), "rows of a K view")


def test_round_f16_is_round_to_nearest_even():
    from unstructured_sparse_skinny_b200 import tp
    g = torch.Generator().manual_seed(238)
    x = torch.cat([torch.randn(1_000_003, generator=g) * 300.0,
                   torch.tensor([65504.0, 65519.99, 65520.0, -65520.0, 1e9, float("inf"), -float("inf"),
                                 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, -0.0, 0.0, 1.0 + 2.0 ** -11])])
    y = tp.round_f16(x.cuda()).cpu()
    fs.check_device_status()
    assert torch.equal(y.view(torch.int16), x.half().view(torch.int16))
    n = torch.tensor([float("nan")] * 9).cuda()
    assert torch.isnan(tp.round_f16(n).float()).all()


def test_k_split_collective_on_one_rank():
    """The K-split baseline through NCCL with one rank: the fp32 partial is the
    whole product, the all-reduce is the identity, and the rounded result is
    the fp16 SpMM's, bit for bit (same plan, same accumulators)."""
    import socket

    import torch.distributed as dist
    from unstructured_sparse_skinny_b200 import tp
    M, K, N = 1536, 2048, 16
    W = synth.sparse_weight(M, K, 80, "uniform", (239, 0))
    B = synth.activations_fp16(N, K, (239, 0))
    t = _encode(W)
    Bd = torch.from_numpy(B).cuda()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    try:
        k0, k1 = tp.shard_range(K, 64, 0, 1)
        C = tp.spmm_lscd_ksplit(t.slice_cols(k0, k1), Bd)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    ref = fs.spmm_lscd(t, Bd)
    fs.check_device_status()
    assert torch.equal(C.view(torch.int16), ref.view(torch.int16))
