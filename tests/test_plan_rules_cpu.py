"""Properties of the decode planner's rules (their Python restatement, which
tests/test_gpu_plan.py holds the GPU planner to bit for bit), on random
page layouts: every tile of the call is covered by exactly one CTA pair's
run; each pair's first stream holds its first tile; when every stream has
the same tile count and the aligned chunk is taken, no run straddles a
stream boundary; the aligned chunk costs at most a quarter more tiles per
pair than the even split."""
import types

import numpy as np
import pytest

from tests.plan_rules import MIN_CHUNK, PAGE, cpu_plan


def _inputs(lengths, s_q=1, max_pages=None, prefix=0):
    B = len(lengths)
    mp = max_pages or max(1, max(-(-(prefix + l) // PAGE) for l in lengths))
    segs = np.zeros((B, 2, 4), np.int32)
    for b, l in enumerate(lengths):
        if prefix:
            segs[b, 0] = (0, prefix, 0, 0)
            segs[b, 1] = (prefix, prefix + l, 1, prefix)
        else:
            segs[b, 0] = (0, l, 0, 0)
    return types.SimpleNamespace(wl=types.SimpleNamespace(B=B, s_q=s_q), segs=segs,
                                 block_table=np.zeros((B, mp), np.int32),
                                 deltas=np.array([0, prefix], np.int32),
                                 gather_rows=None, n_gather=None)


def _check_properties(inp, n_h, G):
    r = cpu_plan(inp, n_h, G)
    U, C, off = r["U"], r["C"], r["off"]
    counts = np.diff(off)
    assert C >= MIN_CHUNK and G * C >= U
    covered = np.zeros(U, int)
    for g in range(G):
        u0, u1 = g * C, min(U, g * C + C)
        if u0 >= U:
            assert r["first"][g] == 0
            continue
        covered[u0:u1] += 1
        s = r["first"][g]
        assert off[s] <= u0 < off[s + 1] and counts[s] > 0
    assert (covered == 1).all()
    even = max(MIN_CHUNK, -(-U // G))
    if C != even:
        T0 = counts[0]
        assert (counts == T0).all() and T0 > 0 and 4 * C <= 5 * even
        for g in range(G):
            u0, u1 = g * C, min(U, g * C + C)
            if u0 >= U:
                continue
            # the run lies inside one stream or is made of whole streams
            assert (u0 // T0 == (u1 - 1) // T0) or (u0 % T0 == 0 and u1 % T0 == 0)
    return r


@pytest.mark.parametrize("seed", range(40))
def test_random_layouts(seed):
    g = np.random.default_rng(seed)
    B = int(g.integers(1, 40))
    s_q = int(g.integers(1, 3))
    n_h = int(g.choice([8, 64, 128, 200]))
    G = int(g.choice([3, 10, 74]))
    if g.random() < 0.5:
        lengths = [int(g.integers(1, 5000))] * B          # equal lengths
    else:
        lengths = [int(x) for x in g.integers(1, 5000, B)]
    prefix = int(g.choice([0, 128, 640]))
    _check_properties(_inputs(lengths, s_q, prefix=prefix), n_h, G)


def test_aligned_chunk_examples():
    # 16 x 4096 rows over 74 pairs: 32 tiles per stream, even split 7, the
    # divisor 8 (4 pairs per sequence) is taken
    r = _check_properties(_inputs([4096] * 16), 128, 74)
    assert r["C"] == 8
    # 100 streams of 2 tiles: the multiple 4 would be more than 5/4 of 3
    r = _check_properties(_inputs([256] * 100), 128, 74)
    assert r["C"] == 3
    # 2 x 262144 rows, two query tokens: 4 streams of 2048 tiles, chunk 128
    r = _check_properties(_inputs([262144] * 2, s_q=2), 128, 74)
    assert r["C"] == 128 and r["n_streams"] == 4
