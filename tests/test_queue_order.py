"""The pass-2 work queue, checked on the host.

Pass 2 is one persistent launch over a queue of work items dealt round-robin
to the SM pairs:

    G(0) | dX(0) dW(0) G(1) | dX(1) dW(1) G(2) | ... | dX(C-1) dW(C-1)

A dW item covers two adjacent 256-column hidden tiles (the last one alone
when their number is odd).  The queue drains only if every tile appears
exactly once and every dependency points to an earlier item.  The
dependencies:
- a dX(c) mainloop waits for its token tile's G(c) row;
- a dX(c) epilogue waits for dX(c-1) of its token tile;
- a dW(c) mainloop waits for its G(c) column;
- a G(c) epilogue waits for dX(c-1) of its token tile and dW(c-1) of its column.

This module restates the kernel's item decoder in Python (the G tiles of a
chunk: the first `cols_first` vocabulary tiles column by column, the rest row
by row) and checks both properties for the workload shapes, the small test
shapes and every G order the library uses."""
import itertools

import pytest

TILE = 256
VC = 2048  # vocabulary entries per chunk


def layout(N, H, V):
    TM, HN, C = -(-N // TILE), -(-H // TILE), -(-V // VC)
    VT_last = -(-(V - (C - 1) * VC) // TILE)
    VTf = VC // TILE if C > 1 else VT_last
    return dict(TM=TM, HN=HN, HW=(HN + 1) // 2, C=C, VTf=VTf, VT_last=VT_last)


def dw_tiles(p, b):
    """Hidden tiles of dW item b: a pair, or the last tile alone."""
    if p["HW"] == p["HN"]:
        return (b,)
    return (2 * b, 2 * b + 1) if 2 * b + 1 < p["HN"] else (2 * b,)


def vtiles(p, c):
    return p["VT_last"] if c == p["C"] - 1 else p["VTf"]


def section_size(p, c):
    n = p["TM"] * p["HN"] + vtiles(p, c) * p["HW"]
    if c + 1 < p["C"]:
        n += vtiles(p, c + 1) * p["TM"]
    return n


def total_items(p):
    return vtiles(p, 0) * p["TM"] + sum(section_size(p, c) for c in range(p["C"]))


def grad_tile(p, c, r, cols_first):
    vt = vtiles(p, c)
    k = min(cols_first, vt)
    head = k * p["TM"]
    if r < head:
        return r % p["TM"], r // p["TM"]          # (token tile, vocabulary tile)
    r2, w = r - head, vt - k
    return r2 // w, k + r2 % w


def decode(p, i, cols_first):
    g0 = vtiles(p, 0) * p["TM"]
    if i < g0:
        return ("G", 0) + grad_tile(p, 0, i, cols_first)
    r, c = i - g0, 0
    while c + 1 < p["C"] and r >= section_size(p, c):
        r -= section_size(p, c)
        c += 1
    nx, nw = p["TM"] * p["HN"], vtiles(p, c) * p["HW"]
    if r < nx:
        return ("X", c, r // p["HN"], r % p["HN"])
    if r < nx + nw:
        r -= nx
        return ("W", c, r // p["HW"], r % p["HW"])
    return ("G", c + 1) + grad_tile(p, c + 1, r - nx - nw, cols_first)


def every_tile(p):
    out = set()
    for c in range(p["C"]):
        for t, v in itertools.product(range(p["TM"]), range(vtiles(p, c))):
            out.add(("G", c, t, v))
        for t, h in itertools.product(range(p["TM"]), range(p["HN"])):
            out.add(("X", c, t, h))
        for v, w in itertools.product(range(vtiles(p, c)), range(p["HW"])):
            out.add(("W", c, v, w))
    return out


def dependencies(p, item):
    k, c, a, b = item
    if k == "X":
        deps = [("G", c, a, v) for v in range(vtiles(p, c))]
        return deps + ([("X", c - 1, a, h) for h in range(p["HN"])] if c else [])
    if k == "W":
        return [("G", c, t, a) for t in range(p["TM"])]
    if c == 0:
        return []
    return [("X", c - 1, a, h) for h in range(p["HN"])] + [("W", c - 1, b, w) for w in range(p["HW"])]


def rows_first(p, pairs=74):
    """The library's choice: row by row when a chunk's G tiles fill at most
    three rounds of the SM pairs."""
    return p["TM"] * p["VTf"] <= 3 * pairs


SHAPES = [
    (256, 256, 4096), (300, 136, 5000), (1, 64, 300), (130, 8, 700), (200, 128, 2), (129, 96, 100),
    (384, 512, 9000), (640, 256, 3000), (256, 4096, 1024), (520, 264, 6208), (1100, 192, 4700),
    (8192, 4096, 128256), (4096, 2304, 256000), (32768, 3072, 32064), (16384, 4096, 128256),
    (1000, 512, 2048), (1000, 512, 4097), (6912, 512, 6144), (7168, 512, 6144),
]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("cols_first", [0, 2, 1 << 20])
def test_queue_holds_every_tile_once_and_dependencies_point_back(shape, cols_first):
    p = layout(*shape)
    T = total_items(p)
    items = [decode(p, i, cols_first) for i in range(T)]
    assert len(set(items)) == T and set(items) == every_tile(p)
    pos = {it: i for i, it in enumerate(items)}
    for it, i in pos.items():
        assert all(pos[d] < i for d in dependencies(p, it)), (shape, it)


def test_row_order_of_the_workloads():
    """Row by row below three rounds of the 74 pairs: the Gemma-like workload
    (16 token tiles x 8 vocabulary tiles = 128 G tiles a chunk) and N up to
    27 token tiles; the Llama head, long context and Phi-3 go column by column."""
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
        t, _ = grad_tile(p, 1, r, 0)
        last[t] = r
    assert [last[t] for t in range(p["TM"])] == [(t + 1) * p["VTf"] - 1 for t in range(p["TM"])]
    last = {}
    for r in range(p["TM"] * p["VTf"]):
        t, _ = grad_tile(p, 1, r, 1 << 20)
        last[t] = r
    assert min(last.values()) == (p["VTf"] - 1) * p["TM"]


@pytest.mark.parametrize("shape", SHAPES)
def test_dw_items_cover_every_hidden_tile_once(shape):
    """The dW items of a vocabulary tile pair the hidden tiles 2b and 2b+1; an
    odd last tile goes alone, and one hidden tile means no pair."""
    p = layout(*shape)
    tiles = [t for b in range(p["HW"]) for t in dw_tiles(p, b)]
    assert tiles == list(range(p["HN"]))
    assert sum(len(dw_tiles(p, b)) == 2 for b in range(p["HW"])) == p["HN"] // 2
