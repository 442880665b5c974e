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

