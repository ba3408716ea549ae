"""The GEMV kernels' K-split plans, read through the workspace query (no GPU).

stq1_gemv_workspace returns 2048 counter bytes plus S * batch * N * 4 bytes of
partial sums when the plan splits K into S > 1 pieces, and 0 otherwise, so the
plan's S can be checked on the host.  Without a device the planner assumes a
148-SM part with 228 KB of shared memory per SM, the B200's figures.
"""

import pytest

import sub_bit_sparse_b200 as stq1


@pytest.fixture
def table_path():
    stq1.set_path(stq1.PATH_TABLE)
    yield
    stq1.set_path(stq1.PATH_AUTO)


@pytest.fixture
def mma_path():
    stq1.set_path(stq1.PATH_MMA)
    yield
    stq1.set_path(stq1.PATH_AUTO)


def _split(n, k, b):
    ws = stq1.LIB.stq1_gemv_workspace(n, k, b)
    if ws == 0:
        return 1
    assert (ws - 2048) % (b * n * 4) == 0
    return (ws - 2048) // (b * n * 4)


@pytest.mark.parametrize("n,k,b,want", [
    (4096, 7168, 1, 14),    # 32 slabs x 14 one-chunk pieces = 448 CTAs (about 3 per SM)
    (4096, 7168, 2, 4),     # two-token units aim at a quarter of the CTAs: 32 x 4, pieces of <= 4 chunks
    (18432, 7168, 2, 1),    # 144 two-token units already exceed that target: no split
    (18432, 7168, 1, 4),    # 144 slabs x 4 pieces (the longest piece of 4 chunks, 14 = 4+4+3+3)
])
def test_split_of_the_benchmark_shapes(table_path, n, k, b, want):
    assert _split(n, k, b) == want


@pytest.mark.parametrize("b", [1, 2, 4, 8])
@pytest.mark.parametrize("n,k", [(4096, 7168), (18432, 7168), (512, 2048), (1000, 4096)])
def test_pieces_are_as_few_as_the_longest_piece_allows(table_path, n, k, b):
    # the plan never uses more pieces than its longest piece needs
    chunks = k // 512
    s = _split(n, k, b)
    assert 1 <= s <= min(chunks, 16)
    longest = -(-chunks // s)
    assert s == -(-chunks // longest)


# Tensor-core decode kernel: (8-token tile, 128-row slab) units, K split in
# whole steps of four blocks (two chunks); the split minimises waves (of two
# CTAs per SM, 296 slots) x steps per piece, ties to fewer pieces.
@pytest.mark.parametrize("n,k,b,want", [
    (4096, 7168, 8, 7),     # 32 units: 7 pieces of one step in one wave (cost 1)
    (4096, 7168, 12, 4),    # 64 units: 4 pieces of 2 steps in one wave (cost 2; 7 pieces take 2 waves)
    (18432, 7168, 8, 2),    # 144 units: 2 pieces of 4 steps in one wave (cost 4) beat 3 pieces in 2 waves (6)
    (512, 2048, 4, 2),      # 4 units, 2 steps
    (37888, 7168, 4, 1),    # 296 units: already two per SM
])
def test_mma_split(mma_path, n, k, b, want):
    s = _split(n, k, b)
    steps = -(-(k // 512) // 2)
    longest = -(-steps // s)
    assert s == -(-steps // longest)      # as few pieces as the longest piece allows
    assert s == want
