"""The decode planner's rules restated in Python (shared by the GPU test that
compares the planner's work list with them bit for bit and by the CPU test
of the rules' own properties).

Per (sequence, query token, 128-head block) stream: its tile count --
ceil(pages / 2) per segment in page mode, ceil(n_gather / 128) for gathered
rows -- or 0 for an invalid sequence; the exclusive prefix sum of the counts;
the chunk C of consecutive tiles per CTA pair (ceil(U / G), at least 1, or
for equal counts T0 > 0 a divisor of T0 with at most G / n_streams parts, or
a multiple of T0 when there are more streams than pairs, taken when it costs
at most a quarter more than the even split); the stream of each pair's first
tile.
"""
import numpy as np

PAGE, TILE, MIN_CHUNK = 64, 128, 1


def seq_plan(inp, b):
    """(tiles, invalid) of sequence b under the planner's rules."""
    segs = inp.segs[b]
    max_pages = inp.block_table.shape[1]
    n_ver = len(inp.deltas)
    tiles, prev_end = 0, 0
    for rb, re, ver, _ in segs:
        if re == rb:
            continue
        if rb < prev_end or re < rb or rb % PAGE or re > max_pages * PAGE or not 0 <= ver < n_ver:
            return 0, True
        prev_end = re
        tiles += (-(-(re - rb) // PAGE) + 1) // 2
    if inp.gather_rows is None:
        return tiles, False
    ng = int(inp.n_gather[b])
    if ng < 0 or ng > inp.gather_rows.shape[1]:
        return 0, True

    def version(r):
        for rb, re, ver, _ in segs:
            if rb <= r < re:
                return ver
        return -1

    g = inp.gather_rows[b]
    for i in range(ng):
        v, v0 = version(g[i]), version(g[i - i % TILE])
        if v < 0 or v != v0:
            return 0, True
    return -(-ng // TILE), False


def cpu_plan(inp, n_h, G):
    n_rt = inp.wl.s_q * -(-n_h // 128)
    counts, bad = [], []
    for b in range(inp.wl.B):
        t, x = seq_plan(inp, b)
        counts += [t] * n_rt
        bad += [int(x)] * n_rt
    n_streams = len(counts)
    off = np.zeros(n_streams + 1, np.int64)
    off[1:] = np.cumsum(counts)
    U = int(off[-1])
    C = max(MIN_CHUNK, -(-U // G))
    T0 = counts[0] if counts else 0
    if T0 > 0 and all(c == T0 for c in counts):
        Ca = 0
        if n_streams > G:
            Ca = T0 * -(-n_streams // G)
        else:
            for parts in range(min(T0, G // n_streams), 0, -1):
                if T0 % parts == 0:
                    Ca = T0 // parts
                    break
        if Ca >= MIN_CHUNK and 4 * Ca <= 5 * C:
            C = Ca

    def stream_of(u):
        lo, hi = 0, n_streams - 1
        while lo < hi:
            mid = (lo + hi + 1) >> 1
            if off[mid] <= u:
                lo = mid
            else:
                hi = mid - 1
        return lo

    first = [stream_of(g * C) if g * C < U else 0 for g in range(G)]
    return dict(U=U, C=C, n_streams=n_streams, off=off, bad=np.array(bad), first=np.array(first))
