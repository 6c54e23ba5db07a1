"""Jagged tile schedule, stated in plain Python -- TEST INFRASTRUCTURE ONLY.

The pages name "tile scheduling" over "jagged sequences" as one of the GDPA
kernel's features (Kunlun paper review, §2.3 "GDPA", last paragraph) without
defining it.  The schedule this library uses, written out:

* ``Lq_b = q_offsets[b+1] - q_offsets[b]``, ``Lk_b`` likewise.
* Query tiles of ``BM`` rows: ``ntile_b = ceil(Lq_b / BM)`` (0 when Lq_b = 0);
  tile ``m`` starts at local row ``m0 = m * BM``.
* The keys a tile can see: ``[lo, hi)`` with ``lo = max(0, m0 - wl)`` when the
  left window is bounded (else 0) and ``hi = min(Lk_b, m0 + BM + wr)`` when
  the right window is bounded (else ``Lk_b``); rounded out to whole key
  blocks of ``BN``: blocks ``[lo // BN, ceil(hi / BN))``, none if hi <= lo.
* The cost of a sample is ``sum over its tiles of (1 + number of key blocks)``.
* ``order`` lists the samples by descending cost, ties by ascending sample
  index (longest-processing-time first; one correct answer, so the GPU
  version is compared bit for bit).
* ``tile_start[p]`` is the number of query tiles of the samples ``order[0..p)``;
  ``tile_start[B]`` is the total number of query tiles.
"""
from __future__ import annotations


def kv_blocks(m0: int, BM: int, Lk: int, BN: int, wl: int, wr: int):
    """Key-block range [first, last) a query tile starting at row m0 may touch."""
    lo = max(0, m0 - wl) if wl >= 0 else 0
    hi = min(Lk, m0 + BM + wr) if wr >= 0 else Lk
    if hi <= lo:
        return 0, 0
    return lo // BN, -(-hi // BN)


def sample_cost(Lq: int, Lk: int, BM: int, BN: int, wl: int, wr: int) -> int:
    ntile = -(-Lq // BM)
    cost = 0
    for m in range(ntile):
        a, b = kv_blocks(m * BM, BM, Lk, BN, wl, wr)
        cost += 1 + (b - a)
    return cost


def tile_schedule(q_offsets, kv_offsets, BM: int, BN: int, wl: int = -1, wr: int = -1):
    """Return (tile_start[B+1], order[B], cost[B]) as Python int lists."""
    qo = [int(x) for x in q_offsets]
    ko = [int(x) for x in kv_offsets]
    B = len(qo) - 1
    cost = []
    ntile = []
    for b in range(B):
        Lq = qo[b + 1] - qo[b]
        Lk = ko[b + 1] - ko[b]
        ntile.append(-(-Lq // BM))
        cost.append(sample_cost(Lq, Lk, BM, BN, wl, wr))
    order = sorted(range(B), key=lambda b: (-cost[b], b))
    tile_start = [0]
    for b in order:
        tile_start.append(tile_start[-1] + ntile[b])
    return tile_start, order, cost
