"""The pass-2 work queue, checked on the host.

Pass 2 is one persistent launch over a queue of work items dealt round-robin
to the SM pairs:

    G(0) | dX(0) dW(0) G(1) | dX(1) dW(1) G(2) | ... | dX(C-1) dW(C-1)

An item is one 256 x 256 tile.  A dW item may pair two adjacent hidden
tiles instead (the last one alone when their number is odd); the library
pairs them when a chunk holds more than three rounds of G tiles for the SM
pairs.  The queue drains only if every tile appears exactly once and every
tile that an item's tiles depend on lies in an earlier item.  The
dependencies:
- a dX(c) mainloop waits for its token tile's G(c) row;
- a dX(c) epilogue waits for dX(c-1) of its token tile;
- a dW(c) mainloop waits for its G(c) column;
- a G(c) epilogue waits for dX(c-1) of its token tile and dW(c-1) of its column.

This module restates the kernel's item decoder in Python (the G columns of a
chunk: the first `cols_first` column by column, the rest row by row) and
checks both properties for the workload shapes, the small test shapes, every
G order and dW items paired or not.  The model can pair G and dX items too
(two vocabulary tiles of a G row, two hidden tiles of a dX row); the queue
drains that way as well, but the library does not pair them: their shorter
contractions measured slower paired."""
import itertools

import pytest

TILE = 256
VC = 2048  # vocabulary entries per chunk


def layout(N, H, V, pair_g=False, pair_x=False, pair_w=False):
    TM, HN, C = -(-N // TILE), -(-H // TILE), -(-V // VC)
    VT_last = -(-(V - (C - 1) * VC) // TILE)
    VTf = VC // TILE if C > 1 else VT_last
    half = (HN + 1) // 2
    return dict(TM=TM, HN=HN, HX=half if pair_x else HN, HW=half if pair_w else HN, pair_g=pair_g, C=C, VTf=VTf,
                VT_last=VT_last)


def vtiles(p, c):
    return p["VT_last"] if c == p["C"] - 1 else p["VTf"]


def gcols(p, c):
    vt = vtiles(p, c)
    return (vt + 1) // 2 if p["pair_g"] else vt


def slot(j, n, tiles):
    """Tiles of item j of n per row, over `tiles` tiles: pairs when n < tiles."""
    if n == tiles:
        return (j,)
    return (2 * j, 2 * j + 1) if 2 * j + 1 < tiles else (2 * j,)


def section_size(p, c):
    n = p["TM"] * p["HX"] + vtiles(p, c) * p["HW"]
    if c + 1 < p["C"]:
        n += gcols(p, c + 1) * p["TM"]
    return n


def total_items(p):
    return gcols(p, 0) * p["TM"] + sum(section_size(p, c) for c in range(p["C"]))


def grad_item(p, c, r, cols_first):
    """(token tile, G column) of the r-th G item of chunk c."""
    gc = gcols(p, c)
    k = min(cols_first, gc)
    head = k * p["TM"]
    if r < head:
        return r % p["TM"], r // p["TM"]
    r2, w = r - head, gc - k
    return r2 // w, k + r2 % w


def decode(p, i, cols_first):
    """Item i as a tuple of the tiles it covers, each (kind, chunk, row, column)."""
    g0 = gcols(p, 0) * p["TM"]

    def grad(c, r):
        t, col = grad_item(p, c, r, cols_first)
        return tuple(("G", c, t, v) for v in slot(col, gcols(p, c), vtiles(p, c)))

    if i < g0:
        return grad(0, i)
    r, c = i - g0, 0
    while c + 1 < p["C"] and r >= section_size(p, c):
        r -= section_size(p, c)
        c += 1
    nx, nw = p["TM"] * p["HX"], vtiles(p, c) * p["HW"]
    if r < nx:
        return tuple(("X", c, r // p["HX"], h) for h in slot(r % p["HX"], p["HX"], p["HN"]))
    if r < nx + nw:
        r -= nx
        return tuple(("W", c, r // p["HW"], h) for h in slot(r % p["HW"], p["HW"], p["HN"]))
    return grad(c + 1, r - nx - nw)


def every_tile(p):
    out = set()
    for c in range(p["C"]):
        for t, v in itertools.product(range(p["TM"]), range(vtiles(p, c))):
            out.add(("G", c, t, v))
        for t, h in itertools.product(range(p["TM"]), range(p["HN"])):
            out.add(("X", c, t, h))
        for v, h in itertools.product(range(vtiles(p, c)), range(p["HN"])):
            out.add(("W", c, v, h))
    return out


def dependencies(p, tile):
    k, c, a, b = tile
    if k == "X":
        deps = [("G", c, a, v) for v in range(vtiles(p, c))]
        return deps + ([("X", c - 1, a, h) for h in range(p["HN"])] if c else [])
    if k == "W":
        return [("G", c, t, a) for t in range(p["TM"])]
    if c == 0:
        return []
    return [("X", c - 1, a, h) for h in range(p["HN"])] + [("W", c - 1, b, h) for h in range(p["HN"])]


def rows_first(p, pairs=74):
    """The library's choice: row by row when a chunk's G tiles fill at most
    three rounds of the SM pairs; items pair their tiles otherwise."""
    return p["TM"] * p["VTf"] <= 3 * pairs


SHAPES = [
    (256, 256, 4096), (300, 136, 5000), (1, 64, 300), (130, 8, 700), (200, 128, 2), (129, 96, 100),
    (384, 512, 9000), (640, 256, 3000), (256, 4096, 1024), (520, 264, 6208), (1100, 192, 4700),
    (8192, 4096, 128256), (4096, 2304, 256000), (32768, 3072, 32064), (16384, 4096, 128256),
    (1000, 512, 2048), (1000, 512, 4097), (6912, 512, 6144), (7168, 512, 6144),
    (7424, 1024, 4100), (7300, 1200, 2300), (7700, 1288, 6200), (8192, 776, 2100),
]
# (G, dX, dW) pairing: the library's two, and the model's other forms
PAIRINGS = [(False, False, False), (False, False, True), (True, True, True)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("cols_first", [0, 2, 1 << 20])
@pytest.mark.parametrize("pairing", PAIRINGS, ids=lambda q: "".join("GXW"[i] if f else "-" for i, f in enumerate(q)))
def test_queue_holds_every_tile_once_and_dependencies_point_back(shape, cols_first, pairing):
    p = layout(*shape, *pairing)
    T = total_items(p)
    items = [decode(p, i, cols_first) for i in range(T)]
    tiles = [t for it in items for t in it]
    assert len(set(tiles)) == len(tiles) and set(tiles) == every_tile(p)
    pos = {t: i for i, it in enumerate(items) for t in it}
    for i, it in enumerate(items):
        for t in it:
            assert all(pos[d] < i for d in dependencies(p, t)), (shape, t)


@pytest.mark.parametrize("shape", SHAPES)
def test_pairs_cover_adjacent_tiles(shape):
    """Paired items hold tiles 2j and 2j+1; an odd last tile goes alone, and
    a row of one tile has no pair."""
    p = layout(*shape, True, True, True)
    for n, tiles in ((p["HX"], p["HN"]), (p["HW"], p["HN"]), (gcols(p, 0), vtiles(p, 0))):
        got = [slot(j, n, tiles) for j in range(n)]
        assert [t for s in got for t in s] == list(range(tiles))
        assert sum(len(s) == 2 for s in got) == (tiles // 2 if n < tiles else 0)


def test_row_order_of_the_workloads():
    """Row by row below three rounds of the 74 pairs: the Gemma-like workload
    (16 token tiles x 8 vocabulary tiles = 128 G tiles a chunk) and N up to
    27 token tiles; the Llama head, long context and Phi-3 go column by column
    and pair their dW items."""
    assert rows_first(layout(4096, 2304, 256000))
    assert rows_first(layout(6912, 4096, 128256))
    assert not rows_first(layout(7168, 4096, 128256))
    for shape in [(8192, 4096, 128256), (16384, 4096, 128256), (32768, 3072, 32064)]:
        assert not rows_first(layout(*shape))


def test_row_order_completes_token_rows_early():
    """What the row order is for: with the G block row by row, token tile t's
    G row is complete after (t + 1) * VT items of the block; column by column
    every row waits for the block's last column."""
    p = layout(4096, 2304, 256000)
    last = {}
    for r in range(p["TM"] * p["VTf"]):
        t, _ = grad_item(p, 1, r, 0)
        last[t] = r
    assert [last[t] for t in range(p["TM"])] == [(t + 1) * p["VTf"] - 1 for t in range(p["TM"])]
    last = {}
    for r in range(p["TM"] * p["VTf"]):
        t, _ = grad_item(p, 1, r, 1 << 20)
        last[t] = r
    assert min(last.values()) == (p["VTf"] - 1) * p["TM"]
