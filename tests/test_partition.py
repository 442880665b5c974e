"""Word-balanced work partition of the automatic SpMM plan, checked on the host
through flashspmm_partition_host (the functions the device kernel runs).

The rule, as the header states it: step q = u * TK + j costs 1024 plus the
words of its two strip tiles; with c(q) the cost of steps [0, q) and P pieces,
bounds[pc] is the smallest q with P * c(q) >= pc * c(T), then raised above its
predecessor and lowered below its successor so that every piece keeps a step.
The restatement below recomputes it with numpy (searchsorted over the full
cost prefix) and must agree entry for entry; the remaining tests check the
properties the SpMM relies on (a strictly increasing cover of [0, T]) and the
balance the table exists for."""
import numpy as np
import pytest

from unstructured_sparse_skinny_b200 import binding
from unstructured_sparse_skinny_b200.build import build_library

STEP_COST = 1024


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build_library()
    binding.load_library()


def tile_words(M, K, kind, seed):
    """Padded word counts of every 64 x 64 tile, [TM, TK], for a few density patterns."""
    g = np.random.default_rng(seed)
    TM, TK = -(-M // 64), -(-K // 64)
    if kind == "uniform":
        w = g.binomial(4096, 0.2, (TM, TK))
    elif kind == "rows":        # strip densities from a heavy-tailed law
        d = np.clip(g.pareto(1.5, TM) * 0.05, 0.0, 1.0)
        w = g.binomial(4096, d[:, None].repeat(TK, 1))
    elif kind == "cols":        # a quarter of the K tiles hot
        d = np.where(g.random(TK) < 0.25, 0.6, 0.07)
        w = g.binomial(4096, d[None, :].repeat(TM, 0))
    elif kind == "spike":       # almost empty, one full tile: the fix-up must keep pieces non-empty
        w = np.zeros((TM, TK), dtype=np.int64)
        w[TM // 2, TK // 2] = 4096
    elif kind == "empty":
        w = np.zeros((TM, TK), dtype=np.int64)
    else:
        raise ValueError(kind)
    return (w + 3) // 4 * 4


def offsets_of(w):
    return np.concatenate([[0], np.cumsum(w.reshape(-1))]).astype(np.int32)


def rule(off, ld, M, K, P):
    """Restatement of the partition rule (numpy, whole cost prefix)."""
    TM, TK = -(-M // 64), -(-K // 64)
    ld = ld or TK
    U = -(-TM // 2)
    T = U * TK
    off = np.asarray(off, dtype=np.int64)
    words = np.zeros((2 * U, TK), dtype=np.int64)    # words of tile (strip, j) of the view
    for s in range(TM):
        row = off[s * ld: s * ld + TK + 1]
        words[s] = np.diff(row)
    step_words = words.reshape(U, 2, TK).sum(axis=1).reshape(-1)
    cost = np.concatenate([[0], np.cumsum(STEP_COST + step_words)])  # c(q), q = 0 .. T
    total = int(cost[-1])
    b = [0] * (P + 1)
    for pc in range(1, P):
        b[pc] = int(np.searchsorted(P * cost, pc * total, side="left"))
    b[P] = T
    for pc in range(1, P):
        b[pc] = max(b[pc], b[pc - 1] + 1)
    for pc in range(P - 1, 0, -1):
        b[pc] = min(b[pc], b[pc + 1] - 1)
    return b, cost


CASES = [(1024, 1024, "uniform"), (4096, 4096, "rows"), (4096, 4096, "cols"), (330, 200, "rows"),
         (12288, 12288, "rows"), (12288, 12288, "cols"), (2048, 8192, "spike"), (640, 576, "empty"),
         (27648, 9216, "uniform"), (100, 64, "uniform")]


@pytest.mark.parametrize("M,K,kind", CASES)
def test_host_rule_matches_restatement(M, K, kind):
    w = tile_words(M, K, kind, seed=M + K)
    off = offsets_of(w)
    TK = -(-K // 64)
    T = -(-(-(-M // 64)) // 2) * TK
    for P in sorted({p for p in (1, 2, 7, min(148, -(-T // 4)), min(T, 300), T) if p <= T}):
        got = binding.partition_host(off, M, K, P)
        want, _ = rule(off, 0, M, K, P)
        assert got == want, (M, K, kind, P)


@pytest.mark.parametrize("M,K,kind", CASES)
def test_table_is_a_strict_cover(M, K, kind):
    w = tile_words(M, K, kind, seed=7 * M + K)
    off = offsets_of(w)
    P = binding.partition_pieces(M, K, 148)
    b = binding.partition_host(off, M, K, P)
    TK = -(-K // 64)
    T = -(-(-(-M // 64)) // 2) * TK
    assert P == binding.plan(M, K, 8, 0, 148)["num_pieces"]
    assert b[0] == 0 and b[-1] == T and len(b) == P + 1
    assert all(b[i] < b[i + 1] for i in range(P))


@pytest.mark.parametrize("M,K,kind", [(4096, 4096, "rows"), (12288, 12288, "rows"), (12288, 12288, "cols"),
                                      (9216, 36864, "rows")])
def test_balance(M, K, kind):
    """No piece costs more than an even share plus one step; even pieces of
    steps do much worse on these skewed matrices."""
    w = tile_words(M, K, kind, seed=3)
    off = offsets_of(w)
    P = binding.partition_pieces(M, K, 148)
    b = binding.partition_host(off, M, K, P)
    _, cost = rule(off, 0, M, K, P)
    per = np.diff(cost[b])
    max_step = int(np.max(np.diff(cost)))
    assert per.max() <= cost[-1] / P + max_step
    T = len(cost) - 1
    even = [pc * T // P for pc in range(P + 1)]
    assert per.max() <= np.diff(cost[even]).max()


def test_uniform_words_give_even_pieces():
    """With the same words in every step the cost is linear in q, so the table
    is the even partition up to rounding."""
    M, K = 9216, 9216
    w = np.full((M // 64, K // 64), 820, dtype=np.int64)
    off = offsets_of(w)
    P = binding.partition_pieces(M, K, 148)
    b = binding.partition_host(off, M, K, P)
    T = (M // 128) * (K // 64)
    assert all(abs(b[pc] - pc * T / P) <= 1 for pc in range(P + 1))


def test_views_follow_their_ld():
    """A K-range view (offsets pointing at K tile j0 with the full matrix's ld)
    and a row view are partitioned over their own steps and words."""
    M, K = 2048, 4096
    w = tile_words(M, K, "rows", seed=11)
    off = offsets_of(w)
    TK = K // 64
    for j0, j1 in ((0, 16), (16, 64), (40, 41)):
        Kv = (j1 - j0) * 64
        P = binding.partition_pieces(M, Kv, 148)
        got = binding.partition_host(off[j0:], M, Kv, P, offsets_ld=TK)
        sub = offsets_of(w[:, j0:j1])           # the same tiles encoded on their own
        assert got == rule(sub, 0, M, Kv, P)[0]
    for i0, i1 in ((0, 8), (8, 32), (31, 32)):
        Mv = (i1 - i0) * 64
        P = binding.partition_pieces(Mv, K, 148)
        got = binding.partition_host(off[i0 * TK:], Mv, K, P, offsets_ld=TK)
        assert got == rule(offsets_of(w[i0:i1]), 0, Mv, K, P)[0]


def test_partition_host_rejects_bad_arguments():
    off = np.zeros(17, dtype=np.int32)
    with pytest.raises(binding.FlashSpmmError):
        binding.partition_host(off, 64, 64, 0)
    with pytest.raises(binding.FlashSpmmError):
        binding.partition_host(off, 64, 1024, 2, offsets_ld=4)   # ld below the 16 tiles per strip
    with pytest.raises(binding.FlashSpmmError):
        binding.partition_host(off, 64, 64, 5)                   # more pieces than steps
