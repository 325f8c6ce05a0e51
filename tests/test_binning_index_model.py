"""CPU model of the cell-route binning's index arithmetic (no GPU).

The kernels in csrc/binsort.cu locate their work through derived indices:
the ranks owning each chunk's first and last pair (recorded by the rank
scan), the window of ranks a 2048-pair tile stages, the walk that generates
the pairs of a tile, the tile mask of a Gaussian inside a 4x4-tile cell, the
segments of a cell list and the (segment, tile) output bases.  This test
restates those rules in Python and checks, on random rectangles, that they
reproduce a direct construction: every generated pair, every chunk
histogram, and the final per-tile lists (rank order) - and that no index
leaves its buffer (staging window <= 2049 ranks, output positions < P).
"""
import random

import numpy as np
import pytest

TILE_KEYS = 2048
CELL = 4
SEG = 1024


def _chunk_size(n, G):
    c = (n + G - 1) // G
    return (c + TILE_KEYS - 1) // TILE_KEYS * TILE_KEYS


def _scene(TX, TY, N, seed):
    rng = np.random.default_rng(seed)
    rects = []
    for _ in range(N):
        if rng.random() < 0.2:
            rects.append(None)
            continue
        big = rng.random() < 0.1
        w = int(rng.integers(1, TX + 1)) if big else int(rng.integers(1, min(3, TX) + 1))
        h = int(rng.integers(1, TY + 1)) if big else int(rng.integers(1, min(3, TY) + 1))
        x0, y0 = int(rng.integers(0, TX - w + 1)), int(rng.integers(0, TY - h + 1))
        rects.append((x0, y0, x0 + w, y0 + h))
    vis = [i for i in range(N) if rects[i]]
    order = [int(g) for g in rng.permutation(vis)]
    return rects, order


def _cell_rect(r):
    x0, y0, x1, y1 = r
    return (x0 // CELL, y0 // CELL, (x1 - 1) // CELL + 1, (y1 - 1) // CELL + 1)


def _owners(off, cnt, P, G):
    """owner_lo / owner_hi per chunk, as the rank scan records them."""
    chunk = _chunk_size(P, G)
    lo_own, hi_own = {}, {}
    for r, (o, n) in enumerate(zip(off, cnt)):
        c = o // chunk
        while c * chunk < o + n and c < G:
            if c * chunk >= o:
                lo_own[c] = r
            last = min((c + 1) * chunk, P) - 1
            if o <= last < o + n:
                hi_own[c] = r
            c += 1
    return chunk, lo_own, hi_own


def _cell_mask(rc, cx, cy):
    x0, y0, x1, y1 = rc
    lx0, lx1 = max(x0 - CELL * cx, 0), min(x1 - CELL * cx, CELL)
    ly0, ly1 = max(y0 - CELL * cy, 0), min(y1 - CELL * cy, CELL)
    if lx1 <= lx0 or ly1 <= ly0:
        return 0
    row = (((1 << (lx1 - lx0)) - 1) << lx0) * 0x1111
    rows = ((1 << (CELL * (ly1 - ly0))) - 1) << (CELL * ly0)
    return row & rows


@pytest.mark.parametrize("TX,TY,N,seed,gmax", [(9, 7, 400, 0, 592), (30, 17, 2500, 1, 592), (4, 4, 50, 2, 592),
                                               (1, 13, 300, 3, 592), (64, 5, 1200, 4, 592),
                                               (120, 68, 12000, 5, 592), (120, 68, 12000, 5, 5)])
def test_cell_route_index_model(TX, TY, N, seed, gmax):
    """gmax caps the CTA count (592 in the library) so that, at sizes Python
    can walk, chunks also span several 2048-pair tiles."""
    rects, order = _scene(TX, TY, N, seed)
    SX, SY = (TX + CELL - 1) // CELL, (TY + CELL - 1) // CELL
    crect = {g: _cell_rect(rects[g]) for g in order}
    cnt = [(crect[g][2] - crect[g][0]) * (crect[g][3] - crect[g][1]) for g in order]
    off = list(np.concatenate([[0], np.cumsum(cnt)[:-1]]).astype(int)) if cnt else []
    P = int(sum(cnt))
    stream = []  # the rank-order cell-pair stream: (cy, cx, g)
    for g in order:
        cx0, cy0, cx1, cy1 = crect[g]
        stream += [(cy, cx, g) for cy in range(cy0, cy1) for cx in range(cx0, cx1)]
    assert len(stream) == P
    G = max(1, min((P + 2047) // 2048, gmax))
    chunk, lo_own, hi_own = _owners(off, cnt, P, G)
    generated = []
    for cta in range(G):
        lo = min(cta * chunk, P)
        hi = min(P, lo + chunk)
        if lo >= hi:
            assert cta not in lo_own
            continue
        # owners equal the searches they replace
        assert lo_own[cta] == max(r for r in range(len(off)) if off[r] <= lo)
        assert hi_own[cta] == max(r for r in range(len(off)) if off[r] <= hi - 1)
        r0, base = lo_own[cta], lo
        while base < hi:
            end = min(base + TILE_KEYS, hi)
            win = [r for r in range(r0, min(len(off), r0 + 9 * 256)) if off[r] < end]
            assert win == list(range(r0, r0 + len(win))) and 1 <= len(win) <= TILE_KEYS + 1
            for q0 in range(0, end - base, 8):  # one thread: 8 consecutive slots
                p = base + q0
                i = max(k for k in range(len(win)) if off[win[k]] <= p)
                g = order[win[i]]
                cx0, cy0, cx1, _ = crect[g]
                w = cx1 - cx0
                local = p - off[win[i]]
                cx, cy = cx0 + local % w, cy0 + local // w
                for j in range(8):
                    if base + q0 + j >= end:
                        break
                    generated.append((cy, cx, g))
                    p += 1
                    if i + 1 < len(win) and off[win[i + 1]] == p:
                        i += 1
                        g = order[win[i]]
                        cx0, cy0, cx1, _ = crect[g]
                        w = cx1 - cx0
                        cx, cy = cx0, cy0
                    else:
                        cx += 1
                        if cx == cx1:
                            cx, cy = cx0, cy + 1
            nx = r0 + len(win)
            r0 = nx if (nx < len(off) and off[nx] == end) else nx - 1
            base = end
    assert generated == stream
    assert G > 1 or P <= 2048
    assert gmax == 592 or chunk > TILE_KEYS  # several tiles per chunk
    # stable sort by cell, segments, counts, bases, expansion
    cells = sorted(range(P), key=lambda i: (stream[i][0] * SX + stream[i][1], i))
    clist = [stream[i] for i in cells]
    T = TX * TY
    tile_cnt = [0] * T
    segs = []
    a = 0
    for c in range(SX * SY):
        b = a
        while b < P and clist[b][0] * SX + clist[b][1] == c:
            b += 1
        for s0 in range(a, b, SEG):
            segs.append((c, s0, min(b, s0 + SEG)))
        a = b
    seg_cnt = []
    for c, s0, s1 in segs:
        cx, cy = c % SX, c // SX
        cc = [0] * 16
        for e in range(s0, s1):
            m = _cell_mask(rects[clist[e][2]], cx, cy)
            assert m
            for bit in range(16):
                cc[bit] += (m >> bit) & 1
        seg_cnt.append(cc)
    seg_base = [None] * len(segs)
    run = {}
    for k, (c, _, _) in enumerate(segs):
        base_c = run.setdefault(c, [0] * 16)
        seg_base[k] = list(base_c)
        run[c] = [x + y for x, y in zip(base_c, seg_cnt[k])]
    for c, tot in run.items():
        cx, cy = c % SX, c // SX
        for bit in range(16):
            tx, ty = CELL * cx + bit % CELL, CELL * cy + bit // CELL
            if tx < TX and ty < TY:
                tile_cnt[ty * TX + tx] = tot[bit]
            else:
                assert tot[bit] == 0
    start = list(np.concatenate([[0], np.cumsum(tile_cnt)[:-1]]).astype(int))
    npairs = int(sum(tile_cnt))
    ids = [None] * npairs
    for k, (c, s0, s1) in enumerate(segs):
        cx, cy = c % SX, c // SX
        nxt = list(seg_base[k])
        for e in range(s0, s1):
            m = _cell_mask(rects[clist[e][2]], cx, cy)
            for bit in range(16):
                if (m >> bit) & 1:
                    tx, ty = CELL * cx + bit % CELL, CELL * cy + bit // CELL
                    pos = start[ty * TX + tx] + nxt[bit]
                    assert 0 <= pos < npairs and ids[pos] is None
                    ids[pos] = clist[e][2]
                    nxt[bit] += 1
    ref = [g for t in range(T) for g in order
           if rects[g][0] <= t % TX < rects[g][2] and rects[g][1] <= t // TX < rects[g][3]]
    assert ids == ref
