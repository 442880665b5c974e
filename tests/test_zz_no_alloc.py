"""The allocation-free SpMM entry point, flashspmm_spmm_lscd_noalloc.

It serves callers that cannot allocate device memory on demand (for example a
plugin inside an engine that owns all device memory, or a latency-critical
path that cannot afford cudaMalloc's implicit synchronisation): its scratch is
a fixed array the library keeps in device memory.  This file is named so that
pytest collects it last; it passes alone in a fresh process and after the
other tests."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import unstructured_sparse_skinny_b200 as fs
from unstructured_sparse_skinny_b200 import binding

pytestmark = pytest.mark.gpu

M, K, N = 4096, 4096, 32


def _problem():
    W = synth.sparse_weight(M, K, 80, "uniform", (300, 0))
    B = synth.activations_fp16(N, K, (300, 0))
    return W, B


def test_noalloc_matches_workspace_entry_point_on_two_calls():
    lib = binding.load_library()
    W, Bh = _problem()
    t = fs.tcsl_encode(torch.from_numpy(W).cuda())
    B = torch.from_numpy(Bh).cuda()
    # this shape is split across pieces, so the scratch array is really used
    assert fs.spmm_workspace_bytes(M, K, N, 0) > 0
    ref = fs.spmm_lscd(t, B)
    fs.check_device_status()
    ref_np = ref.cpu().numpy()
    off, words, _ = oracle.tcsl_encode(W)
    C64, absC, _ = oracle.spmm(off, words, M, K, Bh, nthreads=8)
    assert oracle.tolerance_ok(ref_np, C64, absC).all()  # the workspace entry point itself meets the bound
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        C = torch.full((N, M), float("nan"), dtype=torch.float16, device="cuda")
        v = t.view()
        rc = lib.flashspmm_spmm_lscd_noalloc(ctypes.byref(v), B.data_ptr(), C.data_ptr(), M, K, N, 0, stream)
        assert rc == 0, lib.flashspmm_status_string(rc)
        torch.cuda.synchronize()
        fs.check_device_status()
        out = C.cpu().numpy()
        # against the oracle, with the bound of the parity tests
        ok = oracle.tolerance_ok(out, C64, absC)
        assert ok.all(), f"{int((~ok).sum())} elements outside the bound against the oracle"
        # against the existing entry point: the same bound with its result in
        # the oracle's place, and bit for bit (same plan and kernel)
        ok = oracle.tolerance_ok(out, ref_np.astype(np.float64), absC)
        assert ok.all(), f"{int((~ok).sum())} elements differ from the workspace entry point"
        assert out.tobytes() == ref_np.tobytes()


def test_noalloc_rejects_problems_beyond_the_scratch():
    lib = binding.load_library()
    W, _ = _problem()
    t = fs.tcsl_encode(torch.from_numpy(W).cuda())
    big_n = 256
    assert fs.spmm_workspace_bytes(M, K, big_n, 0) > 16 * 1024 * 1024
    B = torch.zeros((big_n, K), dtype=torch.float16, device="cuda")
    C = torch.zeros((big_n, M), dtype=torch.float16, device="cuda")
    v = t.view()
    rc = lib.flashspmm_spmm_lscd_noalloc(ctypes.byref(v), B.data_ptr(), C.data_ptr(), M, K, big_n, 0,
                                         torch.cuda.current_stream().cuda_stream)
    assert rc == 4  # FLASHSPMM_ERR_CAPACITY, nothing launched
    torch.cuda.synchronize()
    assert (C == 0).all()
