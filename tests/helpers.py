"""Shared helpers for the GPU parity tests: run the CUDA path through the
binding and the oracle on the same seeded inputs."""
import numpy as np
import torch

import oracle
import unstructured_sparse_skinny_b200 as fs


def gpu_encode(W: np.ndarray, tile_m: int = 64, tile_k: int = 64):
    t = fs.tcsl_encode(torch.from_numpy(np.ascontiguousarray(W)).cuda(), tile_m, tile_k)
    fs.check_device_status()
    return t


def gpu_words(t) -> np.ndarray:
    return t.words.cpu().numpy().view(np.uint32)


def assert_encode_bit_exact(W: np.ndarray, tile_m: int = 64, tile_k: int = 64):
    t = gpu_encode(W, tile_m, tile_k)
    off, words, nnz = oracle.tcsl_encode(W, tile_m, tile_k)
    assert np.array_equal(t.tile_offsets.cpu().numpy(), off)
    gw = gpu_words(t)
    assert gw.size == words.size
    assert gw.tobytes() == words.tobytes()
    assert t.nnz == nnz
    return t, off, words


def gpu_spmm(t, B: np.ndarray, split_k: int = 0) -> np.ndarray:
    C = fs.spmm_lscd(t, torch.from_numpy(np.ascontiguousarray(B)).cuda(), split_k=split_k)
    fs.check_device_status()
    return C.cpu().numpy()


def assert_parity(C: np.ndarray, C64: np.ndarray, absC: np.ndarray, what: str = ""):
    ok = oracle.tolerance_ok(C, C64, absC)
    if not ok.all():
        bad = np.argwhere(~ok)
        n, m = bad[0]
        raise AssertionError(f"{what}: {bad.shape[0]} of {ok.size} elements outside tolerance; first at "
                             f"(n={n}, m={m}): gpu={float(C[n, m])!r} oracle={C64[n, m]!r} "
                             f"sum|ab|={absC[n, m]!r}")
