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
