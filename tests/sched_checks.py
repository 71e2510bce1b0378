"""Invariants of the split-KV tile scheduler output.

Any exact cover is a valid schedule, so these checks test properties, not
bytes: every (unit, tile) pair lands in exactly one part, parts are
contiguous, the split counts match the parts that touch each unit, each
piece's workspace slot is unique within its unit, and no part carries much
more than its share of the cost (or, for equal units of more than 64 rows
with two or more parts per unit, every unit is cut into equal pieces of
whole 2-tile steps).
"""
import numpy as np

TILE = 128
OVERHEAD = 3
SPLIT_PENALTY = 8


MAX_ROWS = 128


def units_per_request(s_q, h_q, topk):
    """Paged: the fewest equal blocks of <= 128 rows that cut s_q*h_q rows;
    sparse: one unit per query token."""
    if topk or h_q is None:
        return s_q if topk else 1
    R = s_q * h_q
    n = -(-R // MAX_ROWS)
    while R % n:
        n += 1
    return n


def unit_tiles(seqlens, batch, s_q, topk, h_q=None):
    if topk:
        return [(topk + TILE - 1) // TILE] * (batch * s_q)
    upr = units_per_request(s_q, h_q, topk)
    return [max(0, (int(seqlens[u // upr]) + TILE - 1) // TILE) for u in range(batch * upr)]


def pieces_of_part(md, n):
    """(unit, first tile, end tile, first piece of the part) of each piece."""
    bu, bt, eu, et, first_ws = (int(x) for x in md[:5])
    out = []
    u, t, first = bu, bt, True
    U = len(n)
    while u < U and (u < eu or (u == eu and t < et)):
        tend = min(et, n[u]) if u == eu else n[u]
        if t < tend:
            out.append((u, t, tend, first))
        first = False
        u, t = u + 1, 0
    return out


def rows_per_unit(s_q, h_q, topk):
    """Query rows of one unit; None when h_q is not given."""
    if h_q is None:
        return None
    if topk:
        return h_q
    return s_q * h_q // units_per_request(s_q, h_q, topk)


def equal_unit_pieces(n, parts, rows):
    """Pieces per unit of the equal-unit plan (units of more than 64 rows,
    all with the same tile count n0 > 0, at least two parts per unit):
    k = min(parts // units, ceil(n0 / 2)), or 0 when the cost-axis plan
    applies."""
    U = len(n)
    if rows is None or rows <= 64 or U == 0 or min(n) != max(n) or n[0] <= 0:
        return 0
    k = min(parts // U, (n[0] + 1) // 2)
    return k if k >= 2 else 0


def check_schedule(tile_md, num_splits, seqlens, batch, s_q, topk, parts, h_q=None):
    """h_q=None: one unit per request (s_q*h_q <= 128) on the paged path, with
    at most 64 rows."""
    n = unit_tiles(seqlens, batch, s_q, topk, h_q)
    U = len(n)
    md = np.asarray(tile_md).reshape(parts, 8)
    ptr = np.asarray(num_splits)[:U + 1]
    assert ptr[0] == 0 and np.all(np.diff(ptr) >= 0)
    seen = {}
    touch = [[] for _ in range(U)]
    cost = []
    for p in range(parts):
        pcs = pieces_of_part(md[p], n)
        c = 0
        for (u, t0, t1, first) in pcs:
            for k in range(t0, t1):
                assert (u, k) not in seen, f"tile {(u, k)} in parts {seen[(u, k)]} and {p}"
                seen[(u, k)] = p
            touch[u].append((p, t0, first))
            c += (t1 - t0) + OVERHEAD
        cost.append(c)
    expected = {(u, k) for u in range(U) for k in range(n[u])}
    assert set(seen) == expected, "schedule does not cover every tile exactly once"
    for u in range(U):
        ns = len(touch[u])
        assert ptr[u + 1] - ptr[u] == ns, (u, ptr[u + 1] - ptr[u], ns)
        # the first piece of a unit starts at tile 0, later pieces continue it
        ts = [t0 for (_, t0, _) in touch[u]]
        assert ts == sorted(ts) and (not ts or ts[0] == 0)
        for j, (p, t0, first) in enumerate(touch[u]):
            if ns >= 2:
                ws = int(md[p][4]) if first else int(ptr[u])
                assert ws == ptr[u] + j, (u, p, ws, ptr[u] + j)
    assert ptr[U] <= U + parts
    k = equal_unit_pieces(n, parts, rows_per_unit(s_q, h_q, topk))
    if k:
        # every unit cut into k pieces of whole 2-tile steps, one per part:
        # piece lengths differ by at most one step, later parts are empty
        steps = (n[0] + 1) // 2
        assert list(ptr) == [u * k for u in range(U + 1)]
        for p in range(parts):
            pcs = pieces_of_part(md[p], n)
            if p >= U * k:
                assert pcs == []
                continue
            (u, t0, t1, _), = pcs
            assert u == p // k and t0 % 2 == 0
            assert -(-(t1 - t0) // 2) in (steps // k, -(-steps // k))
        return {"payload": None, "max_cost": max(cost), "splits": int(ptr[U]), "equal_pieces": k}
    total = sum(x + OVERHEAD for x in n if x > 0)
    even = -(-total // parts) if total else 1
    unit_max = max([x + OVERHEAD for x in n if x > 0], default=0)
    # the range grows to the largest unit's cost when that is at most
    # SPLIT_PENALTY tiles above an even share (no split of equal units)
    payload = unit_max if even < unit_max <= even + SPLIT_PENALTY else even
    assert max(cost) <= payload + 2 * OVERHEAD, (max(cost), payload)
    if payload == unit_max and len(set(x for x in n if x > 0)) == 1:
        assert ptr[U] == sum(1 for x in n if x > 0), "equal units must not be split"
    return {"payload": payload, "max_cost": max(cost), "splits": int(ptr[U])}
