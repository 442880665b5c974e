"""The benchmark's multi-rank host logic on CPU ranks (gloo, world size 2):
every rank gets its own, distinct layer (weak scaling, no data exchange), the
reported time is the slowest rank's, and the job throughput counts the bytes
of all ranks.  The SpMM path itself has no collective; the only collectives
are the timing barrier and the max-over-ranks reduction exercised here."""
import os
import socket
import sys
from pathlib import Path

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import bench
    import oracle
    import synth

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        args = bench.parse_args(["--case", "128,256,8,80"])
        calls, _ = bench.workload_calls(args, rank)
        (name, M, K, N, s_pct, structure, key), = calls
        W = synth.sparse_weight(M, K, s_pct, structure, key)
        B = synth.activations_fp16(N, K, key)
        off, words, nnz = oracle.tcsl_encode(W)
        C64, _, _ = oracle.spmm(off, words, M, K, B, nthreads=1)
        local_ms = 10.0 * (rank + 1)  # a stand-in for each rank's device time
        max_ms = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        nbytes = bench.algorithmic_bytes(nnz, M, K, N)
        value = bench.job_throughput(nbytes, 5, max_ms, world)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), key=np.array(key), C=C64, max_ms=max_ms,
                 value=value, nbytes=nbytes)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    r0 = np.load(tmp_path / "rank0.npz")
    r1 = np.load(tmp_path / "rank1.npz")
    assert tuple(r0["key"]) != tuple(r1["key"])          # distinct per-rank seeds
    assert not np.array_equal(r0["C"], r1["C"])          # so distinct problems
    assert float(r0["max_ms"]) == float(r1["max_ms"]) == 20.0  # slowest rank's time on every rank
    expected = world * int(r0["nbytes"]) * 5 / (20.0e-3) / 1e9
    assert abs(float(r0["value"]) - expected) < 1e-9 * expected



def _tp_rank_main(rank: int, world: int, port: int, out_dir: str):
    """Row-split tensor parallelism: every rank holds the same encoded matrix,
    takes its strips through the binding's slicing rule (TCSL.slice_rows), and
    multiplies them with the oracle; the shards are gathered over gloo."""
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import oracle
    import synth
    from unstructured_sparse_skinny_b200.binding import TCSL

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M, K, N = 330, 200, 8  # 6 strips, the last one ragged; ragged K
        W = synth.sparse_weight(M, K, 80, "uniform", (240, 0))  # same matrix on every rank
        B = synth.activations_fp16(N, K, (240, 0))
        off, words, _ = oracle.tcsl_encode(W)
        full = TCSL(torch.from_numpy(off), torch.from_numpy(words.view(np.int32)), 0, M, K)
        strips = -(-M // 64)
        s0, s1 = rank * strips // world, (rank + 1) * strips // world
        shard = full.slice_rows(64 * s0, min(M, 64 * s1))
        C64, _, _ = oracle.spmm(shard.tile_offsets.numpy(), shard.words.numpy().view(np.uint32), shard.M, K, B)
        parts = [None] * world
        dist.all_gather_object(parts, (64 * s0, C64))
        if rank == 0:
            C_full, _, _ = oracle.spmm(off, words, M, K, B)
            C_cat = np.concatenate([c for _, c in sorted(parts, key=lambda x: x[0])], axis=1)
            np.save(os.path.join(out_dir, "tp_ok.npy"), np.array([np.array_equal(C_cat, C_full)]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_row_split(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_tp_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert bool(np.load(tmp_path / "tp_ok.npy")[0])  # the shards' products are the full product's rows


def _ksplit_rank_main(rank: int, world: int, port: int, out_dir: str):
    """K-split tensor parallelism: every rank takes its K range of one encoded
    matrix through the binding's view rule (TCSL.slice_cols) and the shard
    boundaries of unstructured_sparse_skinny_b200.tp, multiplies it with the
    oracle, and the fp64 partials are summed by an all-reduce over gloo."""
    sys.path.insert(0, str(ROOT))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime

    import oracle
    import synth
    from unstructured_sparse_skinny_b200.binding import TCSL
    from unstructured_sparse_skinny_b200.tp import shard_range

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        M, K, N = 330, 968, 8  # ragged strips and a ragged last K tile (968 = 15 * 64 + 8)
        W = synth.sparse_weight(M, K, 80, "power_law", (241, 0))
        B = synth.activations_fp16(N, K, (241, 0))
        off, words, _ = oracle.tcsl_encode(W)
        full = TCSL(torch.from_numpy(off), torch.from_numpy(words.view(np.int32)), 0, M, K)
        k0, k1 = shard_range(K, 64, rank, world)
        view = full.slice_cols(k0, k1)
        # gather the view's tiles through its addressing rule: tile (i, j) at offsets[i * ld + j]
        TM, TKv = -(-M // 64), -(-(k1 - k0) // 64)
        voff, ld = view.tile_offsets.numpy(), view.offsets_ld
        segs = [words[voff[i * ld + j]:voff[i * ld + j + 1]] for i in range(TM) for j in range(TKv)]
        g_off = np.concatenate([[0], np.cumsum([len(x) for x in segs])]).astype(np.int32)
        g_words = np.concatenate(segs) if segs else np.zeros(0, np.uint32)
        s_off, s_words, _ = oracle.tcsl_encode(np.ascontiguousarray(W[:, k0:k1]))
        same = np.array_equal(g_off, s_off) and g_words.tobytes() == s_words.tobytes()
        C64, _, _ = oracle.spmm(g_off, g_words, M, k1 - k0, np.ascontiguousarray(B[:, k0:k1]), nthreads=1)
        part = torch.from_numpy(np.ascontiguousarray(C64))
        dist.all_reduce(part, op=dist.ReduceOp.SUM)
        flags = torch.tensor([1 if same else 0], dtype=torch.int64)
        dist.all_reduce(flags, op=dist.ReduceOp.MIN)
        if rank == 0:
            C_full, absC, _ = oracle.spmm(off, words, M, K, B, nthreads=1)
            err = np.abs(part.numpy() - C_full)
            np.save(os.path.join(out_dir, "ksplit_ok.npy"),
                    np.array([bool(flags.item()), bool((err <= 1e-12 * absC).all()), bool(absC.max() > 0)]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_k_split(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_ksplit_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    views_match, sum_matches, nontrivial = np.load(tmp_path / "ksplit_ok.npy")
    assert views_match     # each rank's K view addresses exactly the tiles of its own encoding
    assert sum_matches     # the all-reduced partials are the full product (fp64, up to summation order)
    assert nontrivial


def test_shard_ranges_cover():
    sys.path.insert(0, str(ROOT))
    from unstructured_sparse_skinny_b200.tp import shard_range
    for extent, world in ((968, 2), (12288, 8), (100, 3), (64, 4)):
        r = [shard_range(extent, 64, k, world) for k in range(world)]
        assert r[0][0] == 0 and r[-1][1] == extent
        assert all(r[k][1] == r[k + 1][0] for k in range(world - 1))
        assert all(b % 64 == 0 for b, _ in r)
