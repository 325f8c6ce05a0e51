"""CPU model of the index arithmetic of the binning and render kernels (no GPU).

The kernels in csrc/binsort.cu locate their work through derived indices:
the ranks owning each chunk's first and last pair (recorded by the rank
scan), the window of ranks a 2048-pair tile stages, the walk that generates
the pairs of a tile, the tile mask of a Gaussian inside a 4x4-tile cell (as the
cell-pair key carries it, from the cell rectangle and 8 bits of offsets), the
segments of a cell list and the (segment, tile) output bases.  This test
restates those rules in Python and checks, on random rectangles, that they
reproduce a direct construction: every generated pair, every chunk
histogram, and the final per-tile lists (rank order) - and that no index
leaves its buffer (staging window <= 2049 ranks, output positions < P).
The render kernels' contribution-mask words (written per staged batch by the
forward, walked back to front by the backward) are modelled the same way.
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


def _sub_offsets(r):
    """The 8-bit offsets of a tile rectangle inside its first and last cells
    (csrc/binsort.cu, sub_offsets)."""
    x0, y0, x1, y1 = r
    return (x0 & 3) | ((x1 - 1) & 3) << 2 | (y0 & 3) << 4 | ((y1 - 1) & 3) << 6


def _cell_pair_key(crect, sb, cx, cy):
    """The cell-pair key with the pair's tile mask in bits 8-15 and 24-31
    (csrc/binsort.cu, cell_pair_key), from the cell rectangle and the
    sub-offsets only."""
    cx0, cy0, cx1, cy1 = crect
    lx0 = sb & 3 if cx == cx0 else 0
    lx1 = (sb >> 2) & 3 if cx == cx1 - 1 else 3
    ly0 = (sb >> 4) & 3 if cy == cy0 else 0
    ly1 = sb >> 6 if cy == cy1 - 1 else 3
    row = ((2 << lx1) - (1 << lx0)) * 0x1111
    rows = (2 << (4 * ly1 + 3)) - (1 << (4 * ly0))
    m = row & rows
    assert 0 <= cx < 256 and 0 <= cy < 256 and 0 < m < (1 << 16)
    return cx | (m & 0xFF) << 8 | cy << 16 | (m >> 8) << 24


def _key_mask(key):
    return ((key >> 8) & 0xFF) | ((key >> 24) << 8)


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
                    # the key carries the cell (the radix digits) and the pair's tile mask
                    key = _cell_pair_key(crect[g], _sub_offsets(rects[g]), cx, cy)
                    assert key & 0x00FF00FF == cy << 16 | cx
                    assert _key_mask(key) == _cell_mask(rects[g], cx, cy)
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


# --------------------------------------------------------------------------
# Render kernels: contribution-mask words and the backward's walk
# --------------------------------------------------------------------------

FWD_BATCH = 128  # staged entries per forward batch
QUADS = 4


def _mask_model(ranges, blended, P):
    """The forward's mask writes as render.cu indexes them: per tile, per
    batch of FWD_BATCH entries starting at the tile's first position, per
    word w of 32 staged entries (k0 = batch start + 32 w), quadrant q ORs its
    32 blend bits shifted by o = k0 % 32 into word (k0 // 32) * 4 + q and, when
    o > 0, the rest into the word four further on - each write only below the
    mask's size 4 * ceil(P / 32)."""
    words = QUADS * ((P + 31) // 32)
    mask = np.zeros(words, np.uint64)
    for t, (s, e) in enumerate(ranges):
        for b in range(s, e, FWD_BATCH):
            for w in range(FWD_BATCH // 32):
                k0 = b + 32 * w
                if k0 >= e:
                    break
                for q in range(QUADS):
                    bw = 0
                    for j in range(32):
                        if k0 + j < e and (k0 + j, q) in blended:
                            bw |= 1 << j
                    if not bw:
                        continue
                    o = k0 & 31
                    wi = (k0 >> 5) * QUADS + q
                    assert wi < words
                    mask[wi] |= (bw << o) & 0xFFFFFFFF
                    if o and wi + QUADS < words:
                        mask[wi + QUADS] |= bw >> (32 - o)
                    elif o:
                        assert (bw >> (32 - o)) == 0  # nothing lost at the end of the mask
    return mask.astype(np.uint32)


def _walk_model(mask, s, wlast, q):
    """Positions the backward visits for quadrant q of a tile starting at s,
    in visiting order, with their slot (lane) in the 32-entry staging."""
    out = []
    k_hi = s + wlast - 1
    for wk in range(k_hi >> 5, (s >> 5) - 1, -1):
        kb = wk << 5
        wi = wk * QUADS + q
        assert wi < len(mask)
        bits = int(mask[wi])
        lo = s - kb if s > kb else 0
        hi = k_hi - kb
        assert 0 <= lo <= 31
        if hi < 31:
            bits &= (2 << hi) - 1
        bits &= ~((1 << lo) - 1) & 0xFFFFFFFF
        while bits:
            l = bits.bit_length() - 1
            bits &= ~(1 << l)
            assert 0 <= l < 32
            out.append((kb + l, l))
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_render_mask_words_and_backward_walk(seed):
    """The forward's mask words equal the direct layout (bit k % 32 of word
    (k // 32) * 4 + quadrant for every blended list position k), and the
    backward visits exactly the blended positions up to the quadrant's last
    contributor, back to front, each from its own staging slot k % 32."""
    rng = np.random.default_rng(seed)
    T = 37
    lens = rng.integers(0, 300, T)
    lens[rng.random(T) < 0.2] = 0
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    ranges = [(int(a), int(a + n)) for a, n in zip(starts, lens)]
    P = int(lens.sum())
    blended = {(k, q) for k in range(P) for q in range(QUADS) if rng.random() < 0.3}
    mask = _mask_model(ranges, blended, P)
    direct = np.zeros(QUADS * ((P + 31) // 32), np.uint32)
    for k, q in blended:
        direct[(k >> 5) * QUADS + q] |= np.uint32(1 << (k & 31))
    np.testing.assert_array_equal(mask, direct)
    for s, e in ranges:
        for q in range(QUADS):
            wlast = int(rng.integers(0, e - s + 1)) if e > s else 0
            if wlast == 0:
                continue
            got = _walk_model(mask, s, wlast, q)
            want = sorted((k for k in range(s, s + wlast) if (k, q) in blended), reverse=True)
            assert [k for k, _ in got] == want
            assert all(l == k % 32 for k, l in got)


# ---------------------------------------------------------------------------
# Dispatch order of the render CTAs (csrc/render.cu, order_by_work): one CTA
# of 32 warps sorts n work counts into decreasing 8-bit classes, with the
# classes and positions of the first 32768 items kept in shared memory.

ORDER_THREADS = 1024
ORDER_WARPS = 32
ORDER_CODES = 256
ORDER_STRIDE = ORDER_CODES + 1
ORDER_CNT = ORDER_WARPS * ORDER_STRIDE
ORDER_STAGE = 32768


def _order_code(w):
    if w < 16:
        return w
    e = w.bit_length() - 1
    return 16 + (e - 4) * 8 + ((w >> (e - 3)) & 7)


def _order_model(work):
    """The kernel's phases warp by warp (lanes of one instruction in lane
    order; the kernel's atomics may take any order, which moves items only
    within their (class, warp) group); asserts that every shared-memory and
    output index stays inside its buffer and that the scan's counter reads
    of one warp instruction fall in distinct banks."""
    n = len(work)
    nc = min(n, ORDER_STAGE)
    code = [_order_code(work[i]) for i in range(nc)]
    cnt = [0] * ORDER_CNT
    rows = (n + 31) // 32
    per_warp = (rows + ORDER_WARPS - 1) // ORDER_WARPS

    def items(w):
        i0 = min(rows, w * per_warp) * 32
        i1 = min(n, min(rows, w * per_warp + per_warp) * 32)
        return range(i0, i1)

    def code_of(i):
        return code[i] if i < nc else _order_code(work[i])

    for w in range(ORDER_WARPS):
        for i in items(w):
            x = w * ORDER_STRIDE + code_of(i)
            assert 0 <= x < ORDER_CNT
            cnt[x] += 1
    per = ORDER_CODES * ORDER_WARPS // ORDER_THREADS

    def flat_addr(f):
        return (f & 31) * ORDER_STRIDE + (ORDER_CODES - 1 - (f >> 5))

    for t0 in range(0, ORDER_THREADS, 32):
        for k in range(per):
            assert len({flat_addr((t0 + l) * per + k) % 32 for l in range(32)}) == 32
    assert sorted(flat_addr(f) for f in range(ORDER_CODES * ORDER_WARPS)) == \
        sorted(w * ORDER_STRIDE + c for w in range(ORDER_WARPS) for c in range(ORDER_CODES))
    run = 0
    for f in range(ORDER_CODES * ORDER_WARPS):
        x = flat_addr(f)
        cnt[x], run = run, run + cnt[x]
    assert run == n
    order = [None] * n
    staged = [None] * ORDER_STAGE
    for w in range(ORDER_WARPS):
        for i in items(w):
            x = w * ORDER_STRIDE + code_of(i)
            pos = cnt[x]
            cnt[x] += 1
            assert 0 <= pos < n
            if pos < ORDER_STAGE:
                assert staged[pos] is None
                staged[pos] = i
            else:
                assert order[pos] is None
                order[pos] = i
    for p in range(nc):
        order[p] = staged[p]
    return order


def test_order_code_is_monotone_and_fits_a_byte():
    prev = -1
    for w in sorted(set(list(range(0, 5000)) + [2 ** k + d for k in range(12, 32) for d in (-1, 0, 1)] + [2 ** 32 - 1])):
        c = _order_code(w)
        assert prev <= c <= 239
        prev = c
    assert _order_code(15) == 15 and _order_code(16) == 16 and _order_code(2 ** 32 - 1) == 239


@pytest.mark.parametrize("n", [1, 31, 33, 1023, 1025, 8160, 32640, 32769, 70001])
def test_order_by_work_is_a_heaviest_first_permutation(n):
    """The output is a permutation of 0 .. n-1 in decreasing work class, for
    sizes that leave warps empty, end in a partial row or pass the
    shared-memory staging."""
    rng = np.random.default_rng(n)
    work = [int(x) for x in rng.integers(0, 400, n)]
    for i in rng.choice(n, size=min(n, 5), replace=False):
        work[int(i)] = int(rng.integers(0, 2 ** 32))
    order = _order_model(work)
    assert sorted(order) == list(range(n))
    codes = [_order_code(work[i]) for i in order]
    assert all(a >= b for a, b in zip(codes, codes[1:]))


PART_UNITS = 2048


@pytest.mark.parametrize("T", [1, 16, 85, 103, 256, 2500, 8160])
def test_backward_order_from_partition_histograms(T):
    """The backward's order (csrc/render.cu, k_bwd_prep): the forward counts
    the quadrants of every partition of 2048 per class; block p starts class
    c after all quadrants of higher classes and after class c's quadrants in
    partitions below p.  The result is a permutation of the 4T quadrants in
    decreasing class, and the histograms fit the block between words 9T and
    GS_ORDER_WORDS(T) = 12T + 256."""
    rng = np.random.default_rng(T)
    n = 4 * T
    work = [int(x) for x in rng.integers(0, 600, n)]
    P = (n + PART_UNITS - 1) // PART_UNITS
    assert 9 * T + P * ORDER_CODES <= 12 * T + 256
    hist = [[0] * ORDER_CODES for _ in range(P)]
    for u in range(n):
        hist[u // PART_UNITS][_order_code(work[u])] += 1
    order = [None] * n
    for p in range(P):
        cur = [0] * ORDER_CODES
        for c in range(ORDER_CODES):
            above = sum(hist[q][c2] for q in range(P) for c2 in range(c + 1, ORDER_CODES))
            cur[c] = above + sum(hist[q][c] for q in range(p))
        for u in range(p * PART_UNITS, min(n, (p + 1) * PART_UNITS)):
            c = _order_code(work[u])
            pos = cur[c]
            cur[c] += 1
            assert 0 <= pos < n and order[pos] is None
            order[pos] = u
    codes = [_order_code(work[u]) for u in order]
    assert all(a >= b for a, b in zip(codes, codes[1:]))


# --- radix pass bases: each scatter CTA derives its own digit bases ---------
SORT_MAX_GRID = 148 * 4
SCAN_GROUP = 32
MAX_GROUPS = (SORT_MAX_GRID + SCAN_GROUP - 1) // SCAN_GROUP


def _chunk_bases_model(hist, totals, gtot, c):
    """chunk_bases as the kernel computes it for CTA c: the digit totals'
    exclusive prefix, the group totals of the whole groups before c's group
    (loop over MAX_GROUPS - 1 slots) and the chunk counts of c's group before
    c (loop over SCAN_GROUP - 1 slots)."""
    radix = hist.shape[1]
    g = c // SCAN_GROUP
    base = np.zeros(radix, dtype=np.int64)
    for d in range(radix):
        pre = 0
        for k in range(MAX_GROUPS - 1):
            if k < g:
                pre += int(gtot[k, d])
        for k in range(SCAN_GROUP - 1):
            cc = g * SCAN_GROUP + k
            if cc < c:
                pre += int(hist[cc, d])
        base[d] = int(totals[:d].sum()) + pre
    return base


@pytest.mark.parametrize("G", [1, 2, 31, 32, 33, 64, 65, 300, SORT_MAX_GRID])
@pytest.mark.parametrize("radix", [128, 256])
def test_chunk_bases_equal_a_scan_over_chunks(G, radix):
    rng = np.random.default_rng(G * 7 + radix)
    hist = rng.integers(0, 50, size=(G, radix)) * (rng.random((G, radix)) < 0.6)
    totals = hist.sum(axis=0)
    gtot = np.zeros((MAX_GROUPS, radix), dtype=np.int64)
    for c in range(G):  # what the histogram kernels accumulate
        gtot[c // SCAN_GROUP] += hist[c]
    # reference: the stable pass's offsets, an exclusive scan in (digit, chunk) order
    flat = hist.T.reshape(-1)
    excl = np.concatenate([[0], np.cumsum(flat)[:-1]]).reshape(radix, G)
    cs = sorted({0, G - 1, G // 2, min(G - 1, SCAN_GROUP), min(G - 1, SCAN_GROUP - 1)}
                | set(int(x) for x in rng.integers(0, G, size=min(G, 12))))
    for c in cs:
        assert np.array_equal(_chunk_bases_model(hist, totals, gtot, c), excl[:, c]), (G, radix, c)
    assert (G - 1) // SCAN_GROUP <= MAX_GROUPS - 1  # every group before the last fits the loop


def _stable_pass(keys, digit, G, tile=TILE_KEYS):
    """One stable radix pass as the scatter kernels run it: chunk c of the
    input (G chunks of whole tiles) goes, tile by tile, to each digit's
    region after every earlier chunk's and tile's keys of that digit.
    Returns the output keys and, per input tile, its regrouped keys with
    their output positions (the order of the kernel's write-out)."""
    n = len(keys)
    chunk = _chunk_size(n, G)
    counts = {}
    for k in keys:
        counts[digit(k)] = counts.get(digit(k), 0) + 1
    base, run = {}, 0
    for d in sorted(counts):
        base[d] = run
        run += counts[d]
    out = [None] * n
    tiles = []
    for c in range(G):
        lo, hi = min(c * chunk, n), min(n, c * chunk + chunk)
        for t0 in range(lo, hi, tile):
            t = keys[t0:min(hi, t0 + tile)]
            regrouped = sorted(range(len(t)), key=lambda q: digit(t[q]))  # stable
            placed = []
            for q in regrouped:
                d = digit(t[q])
                out[base[d]] = t[q]
                placed.append((t[q], base[d]))
                base[d] += 1
            tiles.append(placed)
    return out, tiles


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_cell_ranges_from_the_last_cell_pass(seed):
    """The last cell pass (cy digit) records each cell's [start, end) by an
    atomic min / max at the first and last key of each local run of one cell
    in a tile's regrouped write-out; that equals boundary detection on the
    finished cell-sorted list (what a separate pass over it computed)."""
    rng = np.random.default_rng(seed)
    SX, SY = int(rng.integers(1, 40)), int(rng.integers(1, 20))
    n = int(rng.integers(1, 30000))
    cells = rng.integers(0, SX * SY, size=n)
    keys0 = [int(c % SX) | int(c // SX) << 16 for c in cells]
    G = max(1, min((n + 2047) // 2048, SORT_MAX_GRID))
    by_cx, _ = _stable_pass(keys0, lambda k: k & 0xFF, G)
    final, tiles = _stable_pass(by_cx, lambda k: (k >> 16) & 0xFF, G)
    INF = 0xFFFFFFFF
    rng_min = [INF] * (SX * SY)
    rng_max = [0] * (SX * SY)
    for placed in tiles:
        for q, (k, pos) in enumerate(placed):
            cell = (k >> 16) * SX + (k & 0xFF)
            same = lambda j: 0 <= j < len(placed) and placed[j][0] == k and placed[j][1] == pos + (j - q)
            if not same(q - 1):
                rng_min[cell] = min(rng_min[cell], pos)
            if not same(q + 1):
                rng_max[cell] = max(rng_max[cell], pos + 1)
    ranges = [(a, b) if a < b else (0, 0) for a, b in zip(rng_min, rng_max)]
    direct = [(0, 0)] * (SX * SY)
    for p, k in enumerate(final):
        cell = (k >> 16) * SX + (k & 0xFF)
        if p == 0 or final[p - 1] != k:
            direct[cell] = (p, direct[cell][1])
        if p + 1 == len(final) or final[p + 1] != k:
            direct[cell] = (direct[cell][0], p + 1)
    assert ranges == direct
