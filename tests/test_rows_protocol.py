"""Host checks of the row-split kernel's bookkeeping (csrc/q4_rows.cu), no GPU.

The kernel's integer logic is restated here and checked against the
invariants its correctness rests on:

* the share of 8-row groups per CTA (larger shares first, differing by at
  most one group) and the split of a share into tiles (at most the tallest
  height, taller tiles first, heights differing by one group) cover every
  row exactly once, and a launch needs at most four tile heights (four
  tensor-map pairs);
* round robin: stage i lives in ring slot i mod 16 and is computed by warp
  i mod 8, and the stage that refills a slot belongs to the same warp, so a
  warp's waits on a slot's barrier come in phase order (a parity wait cannot
  alias);
* the per-tile reduction (park the partial tile, count it in, the last of
  the tile's contributors adds all partials in stage order), simulated under
  random interleavings of the warps: no partial of another tile is ever read,
  every tile's sum is exact, and no warp waits forever on the exact count of
  reduced tiles that guards a parking buffer's reuse.
"""
import random

import pytest

from bit_weight_dequant_b200 import inputs

W = 8          # warps per CTA
D = 16         # ring slots
MAX_MAPS = 4   # tensor-map pairs per launch


def cta_share(groups: int, ctas: int, c: int):
    """First group and group count of CTA c (larger shares to low indices)."""
    q, r = divmod(groups, ctas)
    g0 = c * (q + 1) if c < r else r * (q + 1) + (c - r) * q
    return g0, q + (1 if c < r else 0)


def tile_heights(ng: int, gmax: int):
    """Row heights of a CTA's tiles: T = ceil(ng / gmax) tiles, taller first."""
    T = -(-ng // gmax)
    base, extra = divmod(ng, T)
    return [8 * (base + (1 if t < extra else 0)) for t in range(T)]


def max_rows(m_pad: int, bs: int, contig: bool) -> int:
    if m_pad == 32:
        return 32
    if bs == 32:
        return 56
    return 72 if (m_pad == 8 and not contig) else 64


SHAPES = sorted({(c.N, c.K) for wl in inputs.workloads().values() for c in wl.cases} |
                {(1, 256), (7, 512), (12, 2560), (100, 1280), (1190, 768), (4100, 768), (248320, 2560)})


@pytest.mark.parametrize("m_pad,bs,contig", [(8, 64, False), (8, 64, True), (16, 64, False), (8, 32, False),
                                             (32, 64, False)])
@pytest.mark.parametrize("ctas", [1, 3, 37, 148])
def test_partition_and_tiles_cover_every_row(m_pad, bs, contig, ctas):
    gmax = max_rows(m_pad, bs, contig) // 8
    for N, _K in SHAPES:
        groups = -(-N // 8)
        n_ctas = min(ctas, groups)
        heights, next_row, shares = set(), 0, []
        for c in range(n_ctas):
            g0, ng = cta_share(groups, n_ctas, c)
            assert 8 * g0 == next_row, "CTA shares must be contiguous and in order"
            hs = tile_heights(ng, gmax)
            assert sum(hs) == 8 * ng and max(hs) <= 8 * gmax
            assert hs == sorted(hs, reverse=True) and max(hs) - min(hs) <= 8
            heights |= set(hs)
            shares.append(ng)
            next_row += 8 * ng
        assert next_row == 8 * groups
        assert shares == sorted(shares, reverse=True) and max(shares) - min(shares) <= 1
        assert len(heights) <= MAX_MAPS, (N, heights)


def test_round_robin_slots_stay_with_one_warp():
    for n_total in (1, 5, 8, 15, 16, 17, 40, 97, 512):
        for i in range(n_total):
            slot, warp = i % D, i % W
            refill = i + D  # issued by stage i's warp into the slot it frees
            if refill < n_total:
                assert refill % D == slot and refill % W == warp
        # so the fills of slot k are consumed by one warp in stage order:
        # its phase-parity waits see phases n - 1 and n only
        for k in range(D):
            stages = list(range(k, n_total, D))
            assert all(s % W == k % W for s in stages)


def simulate_reduction(S: int, T: int, contig: bool, seed: int):
    """One CTA: T tiles of S k-stages, W warps in random interleaving."""
    rng = random.Random(seed)
    n = T * S
    NB = 2 if contig else 1
    if contig:
        starts = [(n * w) // W for w in range(W + 1)]
        seq = {w: list(range(starts[w], starts[w + 1])) for w in range(W)}
    else:
        starts = None
        seq = {w: list(range(w, n, W)) for w in range(W)}

    def contributors(t):
        f, l = t * S, t * S + S - 1
        if not contig:
            return [(f + c) % W for c in range(min(W, S))]
        owner = lambda u: max(w for w in range(W) if starts[w] <= u and starts[w] < starts[w + 1])
        return [w for w in range(owner(f), owner(l) + 1) if starts[w] != starts[w + 1]]

    park, counter, reduced = {}, [0, 0], [0, 0]
    pos = {w: 0 for w in range(W)}
    pending = {w: None for w in range(W)}
    acc = {w: 0 for w in range(W)}
    sums = {}
    stalls = 0
    while any(pos[w] < len(seq[w]) or pending[w] is not None for w in range(W)):
        w = rng.choice([w for w in range(W) if pos[w] < len(seq[w]) or pending[w] is not None])
        if pending[w] is None:  # compute the warp's next stage
            i = seq[w][pos[w]]
            acc[w] += i + 1
            pos[w] += 1
            nxt = seq[w][pos[w]] if pos[w] < len(seq[w]) else None
            if nxt is None or nxt // S != i // S:
                pending[w] = i // S  # leaving tile i // S: flush it
            continue
        t = pending[w]
        b = t % NB
        if t >= NB and reduced[b] < t // NB:  # the buffer's previous tile is not reduced yet: wait
            stalls += 1
            assert stalls < 100000, "a warp waits forever on the reduced-tile count"
            continue
        park[(b, w)] = (t, acc[w])
        acc[w] = 0
        old = counter[b]
        counter[b] += 1
        members = contributors(t)
        assert w in members
        if old == len(members) - 1:  # last contributor: add the parked partials in stage order
            total = 0
            for m in members:
                tt, v = park[(b, m)]
                assert tt == t, f"read a partial of tile {tt} while reducing tile {t}"
                total += v
            assert total == sum(i + 1 for i in range(t * S, t * S + S))
            sums[t] = total
            counter[b] = 0
            reduced[b] += 1
        pending[w] = None
    assert sorted(sums) == list(range(T))


@pytest.mark.parametrize("contig", [False, True])
@pytest.mark.parametrize("S", [1, 2, 3, 5, 7, 8, 9, 16, 32])
@pytest.mark.parametrize("T", [1, 2, 3, 5, 18])
def test_tile_reduction_under_random_interleavings(contig, S, T):
    for seed in range(12):
        simulate_reduction(S, T, contig, seed)
