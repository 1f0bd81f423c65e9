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
