"""Failure detection without faulting the GPU: a bounded in-kernel wait that
nothing completes must end with FLASHSPMM_ERR_TIMEOUT in the device status word,
and the context must stay usable for the next SpMM."""
import numpy as np
import pytest
import torch

import synth
import unstructured_sparse_skinny_b200 as fs
from unstructured_sparse_skinny_b200 import binding
from tests.helpers import assert_parity, gpu_encode, gpu_spmm
import oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives():
    lib = binding.load_library()
    fs.check_device_status()  # start clean
    s = torch.cuda.current_stream().cuda_stream
    assert lib.flashspmm_selftest_wait_timeout(2000, s) == 0  # 2 ms budget
    with pytest.raises(fs.FlashSpmmError) as e:
        fs.check_device_status()
    assert e.value.status == 7
    fs.check_device_status()  # the status word was cleared by the read
    W = synth.sparse_weight(512, 512, 80, "uniform", (220, 0))
    B = synth.activations_fp16(8, 512, (220, 0))
    off, words, _ = oracle.tcsl_encode(W)
    C64, absC, _ = oracle.spmm(off, words, 512, 512, B)
    assert_parity(gpu_spmm(gpu_encode(W), B), C64, absC, "after timeout")


def test_selftest_rejects_bad_budget():
    lib = binding.load_library()
    assert lib.flashspmm_selftest_wait_timeout(0, None) == 1
    assert lib.flashspmm_selftest_wait_timeout(2_000_000, None) == 1
