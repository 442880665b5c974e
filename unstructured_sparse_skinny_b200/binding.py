"""ctypes binding of libflashspmm (argument marshalling only).

Names follow the C ABI in ``include/flashspmm.h`` and the problem statement of
the Flash-LLM review (section 3, "core formulas": C = A x B with sparse
weights A and dense features B): ``tcsl_encode(A_dense, tile_m, tile_k)`` and
``spmm_lscd(tcsl_A, B, C, M, K, N, split_k, stream)``.

Layouts: A is a row-major ``[M, K]`` fp16 tensor; B is passed as the
contiguous ``[N, K]`` tensor (K x N column-major); C is returned as the
contiguous ``[N, M]`` tensor (M x N column-major).
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, replace
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
_LIB_PATH = _PKG / "libflashspmm.so"
_lib = None

STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "ALIGNMENT", 4: "CAPACITY", 5: "CUDA",
                6: "CORRUPT_FORMAT", 7: "TIMEOUT", 8: "NO_DEVICE"}


class FlashSpmmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)} "
                         f"({_lib.flashspmm_status_string(self.status).decode() if _lib else ''})")


class _TcslView(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("K", ctypes.c_int32), ("tile_m", ctypes.c_int32),
                ("tile_k", ctypes.c_int32), ("nnz", ctypes.c_int64), ("nwords", ctypes.c_int64),
                ("tile_offsets", ctypes.c_void_p), ("words", ctypes.c_void_p), ("offsets_ld", ctypes.c_int64),
                ("piece_bounds", ctypes.c_void_p), ("bounds_pieces", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def load_library():
    """Load libflashspmm.so from the package directory (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not _LIB_PATH.exists():
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m unstructured_sparse_skinny_b200.build`"
                           " (the library has no CPU fallback)")
    lib = ctypes.CDLL(str(_LIB_PATH))
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    VP = ctypes.POINTER(_TcslView)
    sig = {
        "flashspmm_abi_version": (ctypes.c_int, []),
        "flashspmm_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "flashspmm_num_tiles": (I64, [I32, I32, I32, I32]),
        "flashspmm_tcsl_count": (ctypes.c_int, [P, I32, I32, I32, I32, P, P, P]),
        "flashspmm_tcsl_fill": (ctypes.c_int, [P, I32, I32, I32, I32, P, P, I64, P]),
        "flashspmm_tcsl_validate": (ctypes.c_int, [VP, P]),
        "flashspmm_tcsl_reorder_banks": (ctypes.c_int, [P, P, I64, I32, I32, I32, I32, P]),
        "flashspmm_spmm_workspace_bytes": (SZ, [I32, I32, I32, I32]),
        "flashspmm_spmm_lscd": (ctypes.c_int, [VP, P, P, I32, I32, I32, I32, P, SZ, P]),
        "flashspmm_spmm_lscd_f32": (ctypes.c_int, [VP, P, P, I32, I32, I32, I32, P, SZ, P]),
        "flashspmm_partition_pieces": (I32, [I32, I32, I32]),
        "flashspmm_tcsl_partition": (ctypes.c_int, [VP, I32, P, I32, P]),
        "flashspmm_partition_host": (ctypes.c_int, [P, I64, I32, I32, I32, P]),
        "flashspmm_round_f16": (ctypes.c_int, [P, P, I64, P]),
        "flashspmm_spmm_lscd_host": (ctypes.c_int, [VP, P, P, P, P, I32, I32, I32, I32, P, SZ, P]),
        "flashspmm_spmm_lscd_noalloc": (ctypes.c_int, [VP, P, P, I32, I32, I32, I32, P]),
        "flashspmm_get_device_status": (ctypes.c_int, [P]),
        "flashspmm_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_uint32, P]),
        "flashspmm_launch_count": (ctypes.c_uint64, []),
        "flashspmm_plan_query": (ctypes.c_int, [I32, I32, I32, I32, I32, P, P]),
        "flashspmm_predict_us": (ctypes.c_int, [I32, I32, I32, I64, I32, P, P]),
        "flashspmm_prefer_sparse": (ctypes.c_int, [I32, I32, I32, I64, I32]),
        "flashspmm_plan_owner": (ctypes.c_int64, [I32, I32, I32, I32, I32, ctypes.c_int64]),
        "flashspmm_plan_slot": (ctypes.c_int64, [I32, I32, I32, I32, I32, ctypes.c_int64, ctypes.c_int64]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise FlashSpmmError(status, where)


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


@dataclass
class TCSL:
    """A Tiled-CSL matrix resident in device memory, or a view of one."""
    tile_offsets: torch.Tensor  # int32; tile (i, j) starts at tile_offsets[i * ld + j]
    words: torch.Tensor         # int32 storage of the uint32 words [nwords]
    nnz: int                    # stored entries without padding; -1 for a view (not counted)
    M: int
    K: int
    tile_m: int = 64
    tile_k: int = 64
    order: int = 0              # 0: ascending loc in a tile; 1: bank-balanced (word order v2)
    offsets_ld: int = 0         # ld above; 0 = ceil(K / tile_k), a whole matrix
    piece_bounds: torch.Tensor | None = None  # int64 word-balanced piece table (flashspmm_tcsl_partition)

    @property
    def nwords(self) -> int:
        return int(self.words.numel())

    @property
    def ld(self) -> int:
        return self.offsets_ld or -(-self.K // self.tile_k)

    def view(self) -> _TcslView:
        pb = self.piece_bounds
        return _TcslView(self.M, self.K, self.tile_m, self.tile_k, self.nnz, self.nwords,
                         self.tile_offsets.data_ptr(), self.words.data_ptr() if self.nwords else None,
                         self.offsets_ld, pb.data_ptr() if pb is not None else None,
                         pb.numel() - 1 if pb is not None else 0, 0)

    def slice_rows(self, row_begin: int, row_end: int) -> "TCSL":
        """Rows [row_begin, row_end) as a view for row-split (tensor-parallel)
        sharding; nothing is copied.  row_begin must start a strip (a multiple of
        tile_m) and row_end must end one or be M.  The view keeps this matrix's
        words and ld and points its offsets at the first strip of the range."""
        if not (0 <= row_begin < row_end <= self.M) or row_begin % self.tile_m or \
                (row_end % self.tile_m and row_end != self.M):
            raise ValueError("a row slice must start and end on strip boundaries")
        i0 = row_begin // self.tile_m
        return replace(self, tile_offsets=self.tile_offsets[i0 * self.ld:], nnz=-1, M=row_end - row_begin,
                       offsets_ld=self.ld, piece_bounds=None)

    def slice_cols(self, k_begin: int, k_end: int) -> "TCSL":
        """Columns [k_begin, k_end) of A (K tiles of every strip) as a view for
        K-split (row-parallel) sharding; nothing is copied.  k_begin must start
        a K tile and k_end must end one or be K.  The view keeps this matrix's
        words and ld and points its offsets at K tile k_begin / tile_k."""
        if not (0 <= k_begin < k_end <= self.K) or k_begin % self.tile_k or \
                (k_end % self.tile_k and k_end != self.K):
            raise ValueError("a column slice must start and end on K-tile boundaries")
        return replace(self, tile_offsets=self.tile_offsets[k_begin // self.tile_k:], nnz=-1, K=k_end - k_begin,
                       offsets_ld=self.ld, piece_bounds=None)

    def partition(self, num_sms: int = 0, stream=None) -> "TCSL":
        """This matrix with a word-balanced piece table for the automatic SpMM
        plan on num_sms SMs (0 = the current device's), computed on the device."""
        lib = load_library()
        sms = num_sms or torch.cuda.get_device_properties(self.tile_offsets.device).multi_processor_count
        P = int(lib.flashspmm_partition_pieces(self.M, self.K, sms))
        if P < 0:
            raise FlashSpmmError(1, "partition_pieces")
        bounds = torch.empty(P + 1, dtype=torch.int64, device=self.tile_offsets.device)
        plain = replace(self, piece_bounds=None)
        v = plain.view()
        _check(lib.flashspmm_tcsl_partition(ctypes.byref(v), sms, bounds.data_ptr(), P + 1,
                                            _stream_handle(stream)), "tcsl_partition")
        return replace(self, piece_bounds=bounds)


def partition_host(tile_offsets, M: int, K: int, num_pieces: int, offsets_ld: int = 0) -> list:
    """The partition rule run on the host over a host copy of the offsets
    (diagnostics and tests; the device computes the same table)."""
    import numpy as np
    off = np.ascontiguousarray(np.asarray(tile_offsets, dtype=np.int32))
    out = (ctypes.c_int64 * (num_pieces + 1))()
    if load_library().flashspmm_partition_host(off.ctypes.data, offsets_ld, M, K, num_pieces, out) != 0:
        raise FlashSpmmError(1, "partition_host")
    return [int(x) for x in out]


def partition_pieces(M: int, K: int, num_sms: int) -> int:
    return int(load_library().flashspmm_partition_pieces(M, K, num_sms))


def tcsl_encode(A_dense: torch.Tensor, tile_m: int = 64, tile_k: int = 64, stream=None, order: int = 0,
                partition: bool = False) -> TCSL:
    """Encode a row-major fp16 ``[M, K]`` device tensor into Tiled-CSL on the GPU.

    Runs the count pass, reads the word total back (one host sync), allocates
    the words with torch, then runs the fill pass; ``order=1`` adds the
    in-place bank-balanced reordering and ``partition=True`` the word-balanced
    piece table for the current device (both 64 x 64 tiles only)."""
    if order not in (0, 1):
        raise ValueError("order must be 0 (ascending loc) or 1 (bank-balanced)")
    lib = load_library()
    if A_dense.dtype != torch.float16 or A_dense.dim() != 2 or not A_dense.is_cuda:
        raise TypeError("A_dense must be a 2-D float16 CUDA tensor")
    A = A_dense.contiguous()
    M, K = A.shape
    s = _stream_handle(stream)
    nt = lib.flashspmm_num_tiles(M, K, tile_m, tile_k)
    if nt < 0:
        raise FlashSpmmError(1, "tcsl_encode")
    off = torch.empty(nt + 1, dtype=torch.int32, device=A.device)
    nnz = torch.empty(1, dtype=torch.int64, device=A.device)
    _check(lib.flashspmm_tcsl_count(A.data_ptr() if A.numel() else None, M, K, tile_m, tile_k,
                                    off.data_ptr(), nnz.data_ptr(), s), "tcsl_count")
    _check(lib.flashspmm_get_device_status(s), "tcsl_count (device)")  # synchronises the stream
    nwords = int(off[-1].item())
    words = torch.empty(max(nwords, 0), dtype=torch.int32, device=A.device)
    _check(lib.flashspmm_tcsl_fill(A.data_ptr() if A.numel() else None, M, K, tile_m, tile_k, off.data_ptr(),
                                   words.data_ptr() if nwords else None, nwords, s), "tcsl_fill")
    if order == 1:
        _check(lib.flashspmm_tcsl_reorder_banks(off.data_ptr(), words.data_ptr() if nwords else None, nwords, M, K,
                                                tile_m, tile_k, s), "tcsl_reorder_banks")
    t = TCSL(off, words, int(nnz.item()), M, K, tile_m, tile_k, order)
    return t.partition(stream=stream) if partition and M > 0 and K > 0 else t


def tcsl_validate(A: TCSL, stream=None) -> None:
    """Checked mode: raises FlashSpmmError(CORRUPT_FORMAT) if the encoding is invalid."""
    lib = load_library()
    s = _stream_handle(stream)
    v = A.view()
    _check(lib.flashspmm_tcsl_validate(ctypes.byref(v), s), "tcsl_validate")
    _check(lib.flashspmm_get_device_status(s), "tcsl_validate (device)")


def plan(M: int, K: int, N: int, split_k: int, num_sms: int) -> dict:
    """The SpMM work plan for num_sms SMs, computed on the host by the library's
    own partition code (diagnostics; no device needed)."""
    lib = load_library()
    info = (ctypes.c_int64 * 9)()
    if lib.flashspmm_plan_query(M, K, N, split_k, num_sms, info, None) != 0:
        raise FlashSpmmError(1, "plan_query")
    keys = ("TM", "TK", "U", "T", "mode", "split", "num_pieces", "partial_slots", "workspace_bytes")
    out = dict(zip(keys, (int(v) for v in info)))
    ranges = (ctypes.c_int64 * (2 * out["num_pieces"]))()
    lib.flashspmm_plan_query(M, K, N, split_k, num_sms, info, ranges)
    out["ranges"] = [(int(ranges[2 * i]), int(ranges[2 * i + 1])) for i in range(out["num_pieces"])]
    return out


def plan_owner(M: int, K: int, N: int, split_k: int, num_sms: int, q: int) -> int:
    return int(load_library().flashspmm_plan_owner(M, K, N, split_k, num_sms, q))


def plan_slot(M: int, K: int, N: int, split_k: int, num_sms: int, pc: int, u: int) -> int:
    return int(load_library().flashspmm_plan_slot(M, K, N, split_k, num_sms, pc, u))


def predict_us(M: int, K: int, N: int, nnz: int, num_sms: int = 148) -> tuple:
    """(sparse, dense) predicted microseconds of one call (host-side model; see
    flashspmm_predict_us in include/flashspmm.h)."""
    a, b = ctypes.c_double(), ctypes.c_double()
    if load_library().flashspmm_predict_us(M, K, N, nnz, num_sms, ctypes.byref(a), ctypes.byref(b)) != 0:
        raise FlashSpmmError(1, "predict_us")
    return a.value, b.value


def prefer_sparse(M: int, K: int, N: int, nnz: int, num_sms: int = 148) -> bool:
    """True when this library's SpMM is predicted faster than a dense GEMM."""
    r = load_library().flashspmm_prefer_sparse(M, K, N, nnz, num_sms)
    if r < 0:
        raise FlashSpmmError(1, "prefer_sparse")
    return r == 1


def spmm_workspace_bytes(M: int, K: int, N: int, split_k: int = 0) -> int:
    return int(load_library().flashspmm_spmm_workspace_bytes(M, K, N, split_k))


_workspaces: dict = {}


def _workspace(device: torch.device, nbytes: int) -> torch.Tensor | None:
    if nbytes == 0:
        return None
    key = (device.index, )
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        # zeroed once here; every completed call leaves its counters zero again
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def spmm_lscd(tcsl_A: TCSL, B: torch.Tensor, C: torch.Tensor | None = None, M: int | None = None,
              K: int | None = None, N: int | None = None, split_k: int = 0, stream=None,
              workspace: torch.Tensor | None = None) -> torch.Tensor:
    """C = A x B.  B is the contiguous ``[N, K]`` fp16 tensor; returns C as ``[N, M]`` fp16, or
    writes the given C, which may be fp32 (the unrounded accumulators: a K-split shard's partial)."""
    lib = load_library()
    M = tcsl_A.M if M is None else M
    K = tcsl_A.K if K is None else K
    if B.dtype != torch.float16 or B.dim() != 2 or not B.is_cuda or not B.is_contiguous():
        raise TypeError("B must be a contiguous [N, K] float16 CUDA tensor")
    N = B.shape[0] if N is None else N
    if B.shape != (N, K):
        raise ValueError(f"B has shape {tuple(B.shape)}, expected ({N}, {K})")
    if C is None:
        C = torch.empty((N, M), dtype=torch.float16, device=B.device)
    elif C.shape != (N, M) or C.dtype not in (torch.float16, torch.float32) or not C.is_contiguous():
        raise ValueError("C must be a contiguous [N, M] float16 or float32 tensor")
    need = int(lib.flashspmm_spmm_workspace_bytes(M, K, N, split_k))
    if workspace is None:
        workspace = _workspace(B.device, need)
    v = tcsl_A.view()
    fn = lib.flashspmm_spmm_lscd if C.dtype == torch.float16 else lib.flashspmm_spmm_lscd_f32
    _check(fn(ctypes.byref(v), B.data_ptr(), C.data_ptr(), M, K, N, split_k,
                                   workspace.data_ptr() if workspace is not None else None,
                                   workspace.numel() if workspace is not None else 0, _stream_handle(stream)),
           "spmm_lscd")
    return C


def spmm_lscd_host(tcsl_A: TCSL, B_host: torch.Tensor, C_host: torch.Tensor, B_dev: torch.Tensor,
                   C_dev: torch.Tensor, split_k: int = 0, stream=None,
                   workspace: torch.Tensor | None = None) -> None:
    """End-to-end call with host activations: H2D copy of B, SpMM, D2H copy of C (all async on stream)."""
    lib = load_library()
    N, K = B_host.shape
    M = tcsl_A.M
    need = int(lib.flashspmm_spmm_workspace_bytes(M, K, N, split_k))
    if workspace is None:
        workspace = _workspace(B_dev.device, need)
    v = tcsl_A.view()
    _check(lib.flashspmm_spmm_lscd_host(ctypes.byref(v), B_host.data_ptr(), C_host.data_ptr(), B_dev.data_ptr(),
                                        C_dev.data_ptr(), M, K, N, split_k,
                                        workspace.data_ptr() if workspace is not None else None,
                                        workspace.numel() if workspace is not None else 0,
                                        _stream_handle(stream)), "spmm_lscd_host")


def spmm_lscd_noalloc(tcsl_A: TCSL, B: torch.Tensor, C: torch.Tensor | None = None, split_k: int = 0,
                      stream=None) -> torch.Tensor:
    """C = A x B through the allocation-free entry point (library-held scratch).

    For callers that cannot allocate device memory on demand; see
    flashspmm_spmm_lscd_noalloc in include/flashspmm.h for the size limit and
    the rule that overlapping calls on one device must not run concurrently."""
    lib = load_library()
    if B.dtype != torch.float16 or B.dim() != 2 or not B.is_cuda or not B.is_contiguous():
        raise TypeError("B must be a contiguous [N, K] float16 CUDA tensor")
    N, K = B.shape
    M = tcsl_A.M
    if C is None:
        C = torch.empty((N, M), dtype=torch.float16, device=B.device)
    v = tcsl_A.view()
    _check(lib.flashspmm_spmm_lscd_noalloc(ctypes.byref(v), B.data_ptr(), C.data_ptr(), M, K, N, split_k,
                                           _stream_handle(stream)), "spmm_lscd_noalloc")
    return C


def check_device_status(stream=None) -> None:
    """Synchronise the stream and raise if a kernel recorded an error."""
    _check(load_library().flashspmm_get_device_status(_stream_handle(stream)), "device status")


def launch_count() -> int:
    return int(load_library().flashspmm_launch_count())
