"""CPU model of the stream-K partition shared by every product kernel
(q4_gemv_sk, q4_skinny_tc, q4_skinny_f16, the tcgen05 FP4 / bf16 products).

T = row_tiles x nchunks iterations in tile-major order; CTA p of P owns
[T p / P, T (p + 1) / P).  The kernels find a tile's contributors with
owner(i) = ((i + 1) P - 1) / T, write a partial tile to slot 2p when the
segment starts the CTA's range and 2p + 1 otherwise, and the last arriver on
the tile's counter (target q_hi - q_lo) reads the slots back with the test
"it_beg(q) >= first iteration of the tile".  These tests restate that
arithmetic and check its invariants on the plans the library launches and on
random sizes: every iteration has exactly one owner, only a range's first
and last segments can be partial, the reader finds exactly the slots the
writers used, no two partial segments share a slot, and whole tiles have one
contributor.
"""
import random

import pytest


def it_beg(p, T, P):
    return (T * p) // P


def owner(i, T, P):
    return ((i + 1) * P - 1) // T


def segments(p, T, P, nchunks):
    """(tile, first_chunk, length, starts_range) of CTA p's range."""
    b, e = it_beg(p, T, P), it_beg(p + 1, T, P)
    out, c = [], b
    while c < e:
        tile, chunk = divmod(c, nchunks)
        n = min(nchunks - chunk, e - c)
        out.append((tile, chunk, n, c == b))
        c += n
    return out


def check_plan(tiles, nchunks, P):
    T = tiles * nchunks
    assert 1 <= P <= T
    # every iteration has exactly one owner, the one whose range holds it
    for i in range(T):
        q = owner(i, T, P)
        assert it_beg(q, T, P) <= i < it_beg(q + 1, T, P)
    written = {}  # tile -> {slot: writer}
    for p in range(P):
        segs = segments(p, T, P, nchunks)
        for k, (tile, chunk, n, first) in enumerate(segs):
            whole = chunk == 0 and n == nchunks
            if not whole:
                # only the first and the last segment of a range are partial
                assert k == 0 or k == len(segs) - 1
                slot = 2 * p + (0 if first else 1)
                assert slot not in written.setdefault(tile, {})
                written[tile][slot] = p
    for tile in range(tiles):
        q_lo = owner(tile * nchunks, T, P)
        q_hi = owner(tile * nchunks + nchunks - 1, T, P)
        parts = written.get(tile, {})
        if q_lo == q_hi:
            assert not parts  # a whole tile: one contributor, no partial
            continue
        # the last arriver's reconstruction of the slots it must add
        read = {}
        for q in range(q_lo, q_hi + 1):
            fs = it_beg(q, T, P) >= tile * nchunks
            read[2 * q + (0 if fs else 1)] = q
        assert read == parts
        # the counter reaches its target exactly when all have arrived
        assert len(parts) - 1 == q_hi - q_lo


def stream_k_P(T, pmax, min_iters):
    return min(max(1, T // min_iters), pmax)


# (name, out, in, chunk codes) of the shapes the bench and the tests launch
SHAPES = [("8b q/k/v grouped", 4096 + 1024 + 1024, 4096), ("8b o", 4096, 4096),
          ("8b gate/up grouped", 2 * 14336, 4096), ("8b down", 4096, 14336),
          ("70b q", 8192, 8192), ("70b k", 1024, 8192), ("70b gate", 28672, 8192),
          ("70b down", 8192, 28672), ("ragged", 300, 1408)]


@pytest.mark.parametrize("name,out,inn", SHAPES)
@pytest.mark.parametrize("kernel,rt,chunk,pmax,min_iters", [
    ("q4_gemv_sk (2 CTAs/SM)", 128, 256, 296, 2),
    ("q4_skinny_tc NT<=32", 128, 256, 296, 4),
    ("q4_skinny_tc / f16 NT>=64", 128, 256, 148, 4),
    ("fp4_gemm_tc", 128, 512, 148, 4),
    ("bf16_gemm_tc", 128, 128, 148, 4)])
def test_plans_launched(name, out, inn, kernel, rt, chunk, pmax, min_iters):
    tiles = -(-out // rt)
    nchunks = -(-inn // chunk)
    P = stream_k_P(tiles * nchunks, pmax, min_iters)
    check_plan(tiles, nchunks, P)


def test_random_plans():
    rng = random.Random(7)
    for _ in range(400):
        tiles = rng.randint(1, 70)
        nchunks = rng.randint(1, 60)
        T = tiles * nchunks
        P = rng.randint(1, min(T, 300))
        check_plan(tiles, nchunks, P)


def test_owner_formula_is_the_inverse_of_the_split():
    for T in (1, 7, 64, 511, 3584):
        for P in sorted({1, 2, 3, 148, 296, T} & set(range(1, T + 1))):
            starts = [it_beg(p, T, P) for p in range(P + 1)]
            for p in range(P):
                for i in range(starts[p], starts[p + 1]):
                    assert owner(i, T, P) == p


# ---------------------------------------------------------------- clusters
# The B <= 8 kernel's cluster fix-up: P = row_tiles x S, and the S CTAs of
# each row tile (one aligned cluster, rank = p % S) add their partial tiles
# through distributed shared memory.  The kernel relies on every CTA's range
# being one non-empty partial segment of row tile p // S, the ranks of a tile
# covering its chunks in rank order.

def cluster_size(tiles, nchunks, P, pmax, slack=2):
    """The library's candidate: the largest S <= 8 that fits the grid, unless
    its CTAs run more than `slack` chunks beyond the longest stream-K range.
    (On the device it is then taken only if all row_tiles clusters of S CTAs
    are resident at once, else the next smaller S is tried.)"""
    T = tiles * nchunks
    sk_iters = -(-T // P)
    for S in range(8, 1, -1):
        if S > nchunks or tiles * S > pmax:
            continue
        return S if -(-nchunks // S) <= sk_iters + slack else 1
    return 1


def check_cluster_plan(tiles, nchunks, S):
    T, P = tiles * nchunks, tiles * S
    covered = [0] * T
    for p in range(P):
        segs = segments(p, T, P, nchunks)
        assert len(segs) == 1  # one segment: one slot of shared memory
        tile, chunk, n, _ = segs[0]
        assert tile == p // S and n >= 1
        assert not (chunk == 0 and n == nchunks)  # never a whole tile
        for i in range(tile * nchunks + chunk, tile * nchunks + chunk + n):
            covered[i] += 1
        if p % S:  # ranks follow each other along K
            prev = segments(p - 1, T, P, nchunks)[0]
            assert prev[0] == tile and prev[1] + prev[2] == chunk
    assert covered == [1] * T


@pytest.mark.parametrize("name,out,inn", SHAPES)
def test_cluster_plans_launched(name, out, inn):
    tiles, nchunks = -(-out // 128), -(-inn // 256)
    P = stream_k_P(tiles * nchunks, 296, 2)
    S = cluster_size(tiles, nchunks, P, 296)
    if S > 1:
        check_cluster_plan(tiles, nchunks, S)


def whole_tile_grid(tiles, nchunks, P, pmax, slack=3):
    """The library's whole-tile grid (when no cluster plan is taken): one CTA
    per row tile if the tiles fit the grid and a tile is at most `slack`
    chunks longer than the longest stream-K range."""
    return tiles <= pmax and nchunks <= -(-tiles * nchunks // P) + slack


def test_cluster_choice_on_the_8b_layer():
    # q/k/v grouped (48 tiles x 16 chunks), o (32 x 16), down (32 x 56):
    # cluster candidates; gate/up grouped (224 tiles) has none and takes the
    # whole-tile grid (16 chunks against 13); the 70B gate/up (224 x 32
    # chunks, against 25) stays on stream-K
    assert cluster_size(48, 16, 296, 296) == 6
    assert cluster_size(32, 16, 256, 296) == 8
    assert cluster_size(32, 56, 296, 296) == 8
    assert cluster_size(224, 16, 296, 296) == 1
    assert whole_tile_grid(224, 16, 296, 296)
    assert cluster_size(224, 32, 296, 296) == 1 and not whole_tile_grid(224, 32, 296, 296)


def test_cluster_choice_on_the_70b_layer():
    # k_proj / v_proj (8 tiles x 32 chunks, stream-K P = 128): S = 8, 4
    # chunks per CTA against 2; q/k/v grouped (80 x 32, P = 296): S = 3, 11
    # against 9; o_proj (64 x 32): S = 4, 8 against 7; down_proj (64 x 112):
    # 28 against 25 stays on stream-K
    assert cluster_size(8, 32, 128, 296) == 8
    assert cluster_size(80, 32, 296, 296) == 3
    assert cluster_size(64, 32, 296, 296) == 4
    assert cluster_size(64, 112, 296, 296) == 1


@pytest.mark.parametrize("tiles,nchunks", [(224, 16), (1, 1), (150, 3), (296, 9)])
def test_whole_tile_grid_partition(tiles, nchunks):
    """P = row_tiles: CTA p's range is exactly row tile p, so no segment is
    partial and the fix-up never runs."""
    T, P = tiles * nchunks, tiles
    for p in range(P):
        assert segments(p, T, P, nchunks) == [(p, 0, nchunks, True)]
    check_plan(tiles, nchunks, P)


def test_random_cluster_plans():
    rng = random.Random(11)
    for _ in range(300):
        S = rng.randint(2, 8)
        nchunks = rng.randint(S, 80)
        tiles = rng.randint(1, 296 // S)
        check_cluster_plan(tiles, nchunks, S)


# ------------------------------------------- tcgen05 products (FP4, bf16)
def tc_cluster_size(tiles, nchunks, nt, pmax=148, min_iters=4):
    """The FP4 / bf16 products' candidate: only for activation tiles nt >= 64,
    the largest S <= 8 with tiles x S CTAs (one per SM), each CTA's range at
    most 25 % longer than the longest stream-K range.  (On the device it is
    then taken only if all clusters are resident at once.)"""
    if nt < 64:
        return 1
    T = tiles * nchunks
    P = stream_k_P(T, pmax, min_iters)
    sk = -(-T // P)
    for S in range(8, 1, -1):
        if S > nchunks or tiles * S > pmax:
            continue
        return S if -(-nchunks // S) * 4 <= sk * 5 else 1
    return 1


def test_tc_cluster_choice_on_70b_shapes():
    # FP4 chunks are 512 codes, bf16 chunks 128 values; 128-row tiles
    assert tc_cluster_size(64, 56, 128) == 2    # FP4 down_proj, B > 64: 28 against 25
    assert tc_cluster_size(64, 56, 64) == 2     # FP4 down_proj, 33 <= B <= 64
    assert tc_cluster_size(64, 56, 32) == 1     # NT <= 32: stream-K
    assert tc_cluster_size(224, 16, 128) == 1   # FP4 gate_proj: 224 tiles > 148 SMs
    assert tc_cluster_size(64, 224, 128) == 2   # bf16 down_proj: 112 against 97
    assert tc_cluster_size(64, 16, 128) == 2    # FP4 q_proj: 8 against 7


@pytest.mark.parametrize("tiles,nchunks", [(3, 8), (3, 5), (3, 3), (64, 56), (64, 224)])
def test_tc_cluster_partition(tiles, nchunks):
    S = tc_cluster_size(tiles, nchunks, 128)
    assert S > 1
    check_cluster_plan(tiles, nchunks, S)
