"""Work partition (step space -> pieces, one CTA each) and the split-K partial
slot mapping, checked on the host through the library's own partition code
(Flash-LLM review, section 3 tiling and section 5 Reduction kernel): the
pieces tile the step space exactly, the owner of every step is the piece
that holds it, every partial sum a piece writes has its own workspace slot,
and the workspace size covers those slots and one arrival counter per unit."""
import itertools

import pytest

from unstructured_sparse_skinny_b200 import binding
from unstructured_sparse_skinny_b200.build import build_library

SHAPES = [(1024, 1024), (130, 72), (64, 64), (1, 8), (9216, 9216), (27648, 9216), (9216, 36864), (200, 136),
          (4096, 256), (128, 8192), (6000, 64), (49152, 12288)]
SPLITS = [0, 1, 2, 3, 7, 1000]
SMS = [1, 2, 7, 148]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_library()
    binding.load_library()


def _align256(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("M,K", SHAPES)
def test_plan_partitions_step_space(M, K):
    for split_k, sms, N in itertools.product(SPLITS, SMS, (8, 64, 256)):
        pl = binding.plan(M, K, N, split_k, sms)
        TM, TK = -(-M // 64), -(-K // 64)
        U = -(-TM // 2)
        assert (pl["TM"], pl["TK"], pl["U"], pl["T"]) == (TM, TK, U, U * TK)
        T, r = pl["T"], pl["ranges"]
        assert r[0][0] == 0 and r[-1][1] == T
        assert all(b < e for b, e in r)                      # no empty piece
        assert all(r[i][1] == r[i + 1][0] for i in range(len(r) - 1))  # contiguous, no overlap
        if split_k <= 0:
            assert pl["mode"] == 0
            assert pl["num_pieces"] == max(1, min(sms, -(-T // 4)))
            lens = [e - b for b, e in r]
            assert max(lens) - min(lens) <= 1                # even split
        else:
            s = min(split_k, TK)
            assert pl["mode"] == 1 and pl["split"] == s and pl["num_pieces"] == U * s
            for pc, (b, e) in enumerate(r):                  # a piece never leaves its unit
                assert b // TK == (e - 1) // TK == pc // s


@pytest.mark.parametrize("M,K", [(1024, 1024), (130, 72), (9216, 9216), (200, 136), (128, 8192), (6000, 64)])
def test_owner_and_partial_slots(M, K):
    for split_k, sms in itertools.product(SPLITS, SMS):
        N = 16
        pl = binding.plan(M, K, N, split_k, sms)
        T, TK, U, r = pl["T"], pl["TK"], pl["U"], pl["ranges"]
        if pl["mode"] == 0:
            step = max(1, T // 997)
            for q in list(range(0, T, step)) + [T - 1]:
                pc = binding.plan_owner(M, K, N, split_k, sms, q)
                assert r[pc][0] <= q < r[pc][1]
        # every (piece, unit) pair where the piece holds only part of the unit
        # writes a partial sum; those slots must be distinct and in range
        writers = []
        for pc, (b, e) in enumerate(r):
            for u in range(b // TK, (e - 1) // TK + 1):
                seg = (max(b, u * TK), min(e, (u + 1) * TK))
                if seg != (u * TK, (u + 1) * TK):
                    writers.append((pc, u))
        if not writers:
            assert pl["partial_slots"] == 0
            assert pl["workspace_bytes"] == 0
            continue
        slots = [binding.plan_slot(M, K, N, split_k, sms, pc, u) for pc, u in writers]
        assert all(0 <= s < pl["partial_slots"] for s in slots)
        assert len(set(slots)) == len(slots)
        # a fixed 4 KB counter region (never holds partial sums, so it stays zero
        # between calls), then the partial sums; counters that do not fit the
        # region (explicit split-K over more than 1024 units) follow them
        counters = pl["num_pieces"] if pl["mode"] == 0 else U
        expect = 4096 + _align256(pl["partial_slots"] * 128 * N * 4)
        if counters > 1024:
            expect += _align256(counters * 4)
        assert pl["workspace_bytes"] == expect
        if pl["mode"] == 0:
            # a shared unit's counter is indexed by its first piece: distinct per shared unit
            shared = sorted({u for _, u in writers})
            firsts = [binding.plan_owner(M, K, N, split_k, sms, u * TK) for u in shared]
            assert len(set(firsts)) == len(firsts)
            # the pieces that contribute to a unit are exactly the owners of its first..last step
            for u in range(U):
                first = binding.plan_owner(M, K, N, split_k, sms, u * TK)
                last = binding.plan_owner(M, K, N, split_k, sms, u * TK + TK - 1)
                overl = [pc for pc, (b, e) in enumerate(r) if b < (u + 1) * TK and e > u * TK]
                assert overl == list(range(first, last + 1))


def test_plan_rejects_bad_arguments():
    lib = binding.load_library()
    import ctypes
    info = (ctypes.c_int64 * 9)()
    assert lib.flashspmm_plan_query(0, 64, 8, 0, 148, info, None) == -1
    assert lib.flashspmm_plan_query(64, 64, 300, 0, 148, info, None) == -1
    assert lib.flashspmm_plan_query(64, 64, 8, 0, 0, info, None) == -1
    assert binding.plan_owner(1024, 1024, 8, 2, 148, 0) == -1  # mode 1 has no owner query
    assert binding.plan_slot(64, 64, 8, 0, 148, 0, 0) == -1     # one piece: no partial sums
