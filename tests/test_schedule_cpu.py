"""The decode kernel's work schedule, restated on the host: stream-K over the
(weight tile, K stage) units of the first sk_tiles tiles, then whole tiles.
These are the formulas the kernel and decode_schedule() in csrc/gemm.cu use
(CTA ranges, segment slots, the contributor range c0..c1 of a tile that the
completing CTA sums); the test checks that every unit is covered exactly
once, that a tile's contributors are exactly c0..c1, that slots stay below
the partial-slot count the workspace is sized for, and that work is balanced.
"""
import itertools

import pytest


def max_seg(units, G, ks):
    if units == 0:
        return 1
    span = (units + G - 1) // G
    return (span - 1) // ks + 2


def schedule(tiles, ks, sms):
    units = tiles * ks
    G = min(units, sms)
    if tiles <= G:
        sk = tiles
    else:
        sk = tiles % G
        if sk > 0 and sk * ks < 2 * G:
            sk += G
    return G, sk, max_seg(sk * ks, G, ks)


def segments(c, G, sk, ks, tiles):
    units = sk * ks
    ub, ue = c * units // G, (c + 1) * units // G
    u, out = ub, []
    while u < ue:
        tm, kb = divmod(u, ks)
        ke = min(ks, kb + ue - u)
        out.append((tm, kb, ke, tm - ub // ks))
        u += ke - kb
    t = sk + c
    while t < tiles:
        out.append((t, 0, ks, 0))
        t += G
    return out


CASES = list(itertools.product([1, 2, 3, 7, 37, 74, 148, 149, 224, 300, 444, 4096], [1, 2, 3, 32, 33], [3, 74, 148]))


@pytest.mark.parametrize("tiles,ks,sms", CASES)
def test_decode_schedule_covers_every_unit_once(tiles, ks, sms):
    G, sk, ms = schedule(tiles, ks, sms)
    units = sk * ks
    cover, load = {}, []
    for c in range(G):
        segs = segments(c, G, sk, ks, tiles)
        load.append(sum(ke - kb for _, kb, ke, _ in segs))
        for tm, kb, ke, slot in segs:
            if not (kb == 0 and ke == ks):          # a partial: needs a slot and a reducer
                assert 0 <= slot < ms
                x0, x1 = tm * ks, tm * ks + ks - 1
                c0 = ((x0 + 1) * G - 1) // units
                c1 = ((x1 + 1) * G - 1) // units
                assert c0 <= c <= c1
                assert slot == tm - (c * units // G) // ks   # the reducer's slot formula
            for k in range(kb, ke):
                assert (tm, k) not in cover
                cover[(tm, k)] = c
    assert len(cover) == tiles * ks
    for tm in range(sk):
        cs = sorted({cover[(tm, k)] for k in range(ks)})
        x0, x1 = tm * ks, tm * ks + ks - 1
        assert cs == list(range(((x0 + 1) * G - 1) // units, ((x1 + 1) * G - 1) // units + 1))
    assert max(load) - min(load) <= ks + 1   # whole tiles differ by at most one per CTA


def test_partial_slots_fit_the_static_scratch_on_148_sms():
    worst = max(schedule(t, ks, 148)[2] for t in range(1, 4097) for ks in (1, 2, 3, 7, 16, 32, 33, 64, 128))
    assert worst <= 3
    assert 65536 + 148 * worst * 16 * 128 * 4 <= 4 << 20   # counters + partials within 4 MiB


def test_headline_decode_shape():
    # 224 weight tiles x 32 stages on 148 SMs: 76 stream-K tiles, then one
    # whole tile per CTA; 48-49 stages each
    G, sk, ms = schedule(224, 32, 148)
    assert (G, sk, ms) == (148, 76, 2)
    loads = [sum(ke - kb for _, kb, ke, _ in segments(c, G, sk, 32, 224)) for c in range(G)]
    assert min(loads) == 48 and max(loads) == 49


# ---------------------------------------------------------------------------
# The prefill (pair) kernel's work items, restated: tiles dealt to the CTA
# pairs round-robin; when the last wave has R < pairs tiles and 2R <= pairs,
# those R tiles run as 2R column halves (launch_pair and locate() in
# csrc/gemm.cu).
# ---------------------------------------------------------------------------
def pair_launch(tiles, max_pairs, single_problem=True):
    rem = tiles % max_pairs
    split = single_problem and rem > 0 and 2 * rem <= max_pairs
    split_from = tiles - rem if split else tiles
    items = tiles + (rem if split else 0)
    npairs = min(items, max_pairs)
    return split_from, items, npairs


def pair_locate(t, split_from):
    if t < split_from:
        return t, 0
    return split_from + ((t - split_from) >> 1), 1 + ((t - split_from) & 1)


@pytest.mark.parametrize("tiles", [1, 2, 5, 33, 37, 38, 73, 74, 75, 88, 110, 111, 112, 148, 256, 1024, 3584])
@pytest.mark.parametrize("max_pairs", [74, 66, 1])
def test_pair_items_cover_every_tile_once(tiles, max_pairs):
    split_from, items, npairs = pair_launch(tiles, max_pairs)
    seen = {}
    per_pair = []
    for pair in range(npairs):
        mine = list(range(pair, items, npairs))
        per_pair.append(mine)
        for t in mine:
            ft, nh = pair_locate(t, split_from)
            assert 0 <= ft < tiles
            key = (ft, nh)
            assert key not in seen, "work item computed twice"
            seen[key] = pair
    for ft in range(tiles):
        whole = (ft, 0) in seen
        halves = (ft, 1) in seen and (ft, 2) in seen
        assert whole != halves, "tile %d: whole=%s halves=%s" % (ft, whole, halves)
        assert ((ft, 1) in seen) == ((ft, 2) in seen)
        if halves:
            assert seen[(ft, 1)] != seen[(ft, 2)], "both halves on one pair"
            assert ft >= tiles - tiles % max_pairs, "only the last wave is split"
    # every pair runs the same number of whole tiles, at most one half tile,
    # and the half tiles come last
    full_rounds = split_from // npairs if npairs else 0
    for mine in per_pair:
        halves = [t for t in mine if t >= split_from]
        assert len(halves) <= 1
        assert len(mine) - len(halves) in (full_rounds, full_rounds + (1 if split_from % npairs else 0))
        assert all(t >= split_from for t in mine[len(mine) - len(halves):])


def test_pair_split_cases():
    # 4096^2 (16 x 16 tiles) on 74 pairs: 34 leftover tiles -> 68 halves
    assert pair_launch(256, 74) == (222, 290, 74)
    # 8192 x 28672: 32 x 112 = 3584 tiles, 32 left -> split
    assert pair_launch(3584, 74)[0] == 3552
    # 8192 x 8192: 1024 tiles, 62 left > 37 -> no split
    assert pair_launch(1024, 74) == (1024, 1024, 74)
    # fewer tiles than half the pairs: every tile split, one half per pair
    assert pair_launch(5, 74) == (0, 10, 10)
    # grouped launches never split
    assert pair_launch(256, 74, single_problem=False)[0] == 256


# The pair kernel's tile order (locate() in csrc/gemm.cu): groups of rg
# consecutive M tiles sweep the N tiles together, M fastest inside a group;
# rg is chosen on the host (fill_pair_problem): all M tiles when A fits in
# 64 MB, else as many as put about 32 MB of A rows in a group.
def raster(lt, tiles_m, tiles_n, rg):
    span = rg * tiles_n
    grp, i = divmod(lt, span)
    m0 = grp * rg
    gm = min(tiles_m - m0, rg)
    return m0 + i % gm, i // gm


def raster_group(M, K, block):
    tiles_m = (M + 255) // 256
    a_tile = 256 * (K // 2 + K // block)
    rg = tiles_m
    if a_tile * tiles_m > (64 << 20):
        rg = ((32 << 20) + a_tile // 2) // a_tile
    return max(1, min(tiles_m, rg))


@pytest.mark.parametrize("tiles_m,tiles_n", [(1, 1), (1, 7), (5, 1), (16, 16), (32, 112), (32, 32), (13, 9), (33, 5)])
@pytest.mark.parametrize("rg", [1, 3, 8, 16, 32, 64])
def test_raster_is_a_bijection(tiles_m, tiles_n, rg):
    rg = min(rg, tiles_m)
    seen = set()
    for lt in range(tiles_m * tiles_n):
        tm, tn = raster(lt, tiles_m, tiles_n, rg)
        assert 0 <= tm < tiles_m and 0 <= tn < tiles_n
        seen.add((tm, tn))
    assert len(seen) == tiles_m * tiles_n
    if rg == tiles_m:   # one group: the plain M-fastest order
        assert all(raster(lt, tiles_m, tiles_n, rg) == (lt % tiles_m, lt // tiles_m)
                   for lt in range(tiles_m * tiles_n))


def test_raster_groups_for_the_bench_shapes():
    # 8192 x 28672 x 8192 and 4096^3: A fits in L2, the order stays M-fastest
    assert raster_group(8192, 8192, 16) == 32
    assert raster_group(4096, 4096, 32) == 16
    # 8192 x 8192 x 28672: 4.1 MB of A per M tile (132 MB in all), 8 per group
    assert raster_group(8192, 28672, 16) == 8
    # a wave of 74 consecutive tiles then touches at most 8 M tiles
    tms = {raster(lt, 32, 32, 8)[0] for lt in range(74)}
    assert len(tms) <= 8
