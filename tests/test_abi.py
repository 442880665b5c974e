"""C-ABI checks that need no GPU: the library builds for sm_100a, loads, exports
every symbol the header declares, and rejects bad arguments on the host
before touching a device."""
import ctypes
import re
from pathlib import Path

import pytest

from unstructured_sparse_skinny_b200 import binding
from unstructured_sparse_skinny_b200.build import build_library

ROOT = Path(__file__).resolve().parent.parent
HEADER = ROOT / "include" / "flashspmm.h"


@pytest.fixture(scope="module")
def lib():
    build_library()
    return binding.load_library()


def declared_symbols():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flashspmm_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_entry_points():
    syms = declared_symbols()
    for s in ("flashspmm_tcsl_count", "flashspmm_tcsl_fill", "flashspmm_spmm_lscd",
              "flashspmm_spmm_workspace_bytes", "flashspmm_get_device_status", "flashspmm_tcsl_validate"):
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_library_is_built_for_sm100a(lib):
    """The build compiles every source for sm_100a only (no PTX for other targets)."""
    from unstructured_sparse_skinny_b200 import build
    flags = " ".join(build.NVCC_FLAGS)
    assert "-gencode arch=compute_100a,code=sm_100a" in flags
    assert flags.count("-gencode") == 1
    assert binding._LIB_PATH.stat().st_mtime >= max(p.stat().st_mtime for p in build.SOURCES)


def test_status_strings_and_version(lib):
    assert lib.flashspmm_abi_version() == 2
    for code in range(9):
        assert lib.flashspmm_status_string(code)
    assert lib.flashspmm_status_string(99) == b"unknown status"


def test_num_tiles(lib):
    assert lib.flashspmm_num_tiles(1024, 1024, 64, 64) == 256
    assert lib.flashspmm_num_tiles(130, 70, 64, 64) == 6
    assert lib.flashspmm_num_tiles(0, 64, 64, 64) == 0
    assert lib.flashspmm_num_tiles(-1, 64, 64, 64) == -1


def _view(**kw):
    v = dict(M=128, K=128, tile_m=64, tile_k=64, nnz=0, nwords=16, tile_offsets=0x10000, words=0x20000)
    v.update(kw)
    return binding._TcslView(**v)


FAKE = 0x7F0000000000  # never dereferenced: every case below fails a host-side check first


@pytest.mark.parametrize("kw,args,status", [
    ({}, dict(M=64), 1),                       # view M != M
    (dict(tile_m=32), {}, 2),                  # SpMM needs 64 x 64 tiles
    ({}, dict(N=300), 2),                      # N > 256
    (dict(K=100), dict(K=100), 2),             # K % 8 != 0
    (dict(words=0x20004), {}, 3),              # misaligned words
    (dict(nwords=6), {}, 6),                   # word count not a multiple of 4
    (dict(tile_offsets=None), {}, 1),          # missing offsets
    (dict(tile_m=256, tile_k=256), {}, 2),     # tile area > 65535
    (dict(offsets_ld=1), {}, 1),               # offsets ld below the tiles per strip (2)
    (dict(offsets_ld=-2), {}, 1),              # negative ld
    (dict(reserved=1), {}, 1),                 # reserved field set
    (dict(piece_bounds=0x30000), {}, 1),       # a piece table without its piece count
    (dict(bounds_pieces=-1), {}, 1),           # negative piece count
])
def test_spmm_rejects_bad_arguments(lib, kw, args, status):
    v = _view(**kw)
    a = dict(M=128, K=128, N=8)
    a.update(args)
    rc = lib.flashspmm_spmm_lscd(ctypes.byref(v), FAKE, FAKE, a["M"], a["K"], a["N"], 0, None, 0, None)
    assert rc == status
    rc = lib.flashspmm_spmm_lscd_f32(ctypes.byref(v), FAKE, FAKE, a["M"], a["K"], a["N"], 0, None, 0, None)
    assert rc == status


def test_partition_and_validate_reject_bad_arguments(lib):
    v = _view()
    assert lib.flashspmm_tcsl_partition(ctypes.byref(v), 148, None, 8, None) == 1       # no table
    assert lib.flashspmm_tcsl_partition(ctypes.byref(_view(tile_k=32)), 148, FAKE, 8, None) == 2
    assert lib.flashspmm_tcsl_partition(ctypes.byref(v), -1, FAKE, 8, None) == 1
    assert lib.flashspmm_tcsl_validate(ctypes.byref(_view(offsets_ld=4)), None) == 2   # views are not validated
    assert lib.flashspmm_partition_pieces(0, 64, 148) == -1
    assert lib.flashspmm_partition_pieces(128, 128, 0) == -1



@pytest.mark.parametrize("args,status", [
    (dict(tile_k=12), 2), (dict(K=100), 2), (dict(tile_m=0), 1), (dict(M=-1), 1),
    (dict(tile_m=256, tile_k=256), 2), (dict(A=FAKE + 8), 3),
])
def test_encoder_rejects_bad_arguments(lib, args, status):
    a = dict(A=FAKE, M=128, K=128, tile_m=64, tile_k=64)
    a.update(args)
    rc = lib.flashspmm_tcsl_count(a["A"], a["M"], a["K"], a["tile_m"], a["tile_k"], FAKE, FAKE, None)
    assert rc == status


def test_null_view_is_invalid(lib):
    assert lib.flashspmm_spmm_lscd(None, FAKE, FAKE, 64, 64, 8, 0, None, 0, None) == 1
    assert lib.flashspmm_tcsl_validate(None, None) == 1


def test_no_device_reported_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    v = _view()
    assert lib.flashspmm_spmm_lscd(ctypes.byref(v), FAKE, FAKE, 128, 128, 8, 0, None, 0, None) == 8
    assert lib.flashspmm_get_device_status(None) == 8
