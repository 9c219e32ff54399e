"""A CPU model of the Hessian kernel's work split (a test of the index arithmetic
only, no GPU): the band edges (128-token tiles for one group; each group charged 64
tokens of work for grouped X), the pieces each CTA walks, their roles and part slots,
the ready flags (including those of bands left without tokens), and the last band's
sums. For random, ragged, piled-up and out-of-order offsets it checks that every
index stays in its buffer, that every token of every group is read once per slab,
that a CTA waits only for flags that a CTA with a lower block index sets, and that
every part written is read exactly once. The constants mirror csrc/hessian.cu.
"""
import numpy as np
import pytest

import synth

SLAB = 128            # channels per CTA slab
STAGE = 128           # tokens per tile
MAX_CTAS = 320        # the grid the workspace is sized for
HEADER = 256          # workspace header bytes
PART_FLOATS = 8 * 256  # one slab's 8 blocks of 16 x 16
MIN_BAND_TILES = 4
GROUP_COST = 64

OWNED, MIDDLE, FIRST_BAND, LAST_BAND = 0, 1, 2, 3


def make_grid(n, c_in, cap):
    slabs = (c_in + SLAB - 1) // SLAB
    sgroups = min(slabs, cap)
    tiles = (n + STAGE - 1) // STAGE
    bmax = max(1, min(cap // sgroups, tiles))
    per = max(MIN_BAND_TILES, (tiles + bmax - 1) // bmax)
    bands = max(1, (tiles + per - 1) // per)
    return slabs, sgroups, bands


def ws_layout(slabs, bands):
    pairs = bands * slabs if bands > 1 else 0
    flag_off = HEADER
    part_off = flag_off + (8 * 2 * 4 * pairs + 255) // 256 * 256
    return flag_off, part_off, part_off + 4 * PART_FLOATS * 2 * pairs


def clamp(x, lo, hi):
    return min(max(x, lo), hi)


def check(n, c_in, offsets, cap, strict=True):
    slabs, sgroups, bands = make_grid(n, c_in, cap)
    ws_slabs, _, ws_bands = make_grid(n, c_in, MAX_CTAS)
    flag_off, part_off, total = ws_layout(ws_slabs, ws_bands)
    G = len(offsets) - 1 if offsets is not None else 1
    C = GROUP_COST if offsets is not None else 0
    ctot = n + C * G

    def hi_of(g):
        return clamp(int(offsets[g + 1]), 0, n)

    def group_range(g):
        if offsets is None:
            return 0, n
        lo = clamp(int(offsets[g]), 0, n)
        return lo, clamp(int(offsets[g + 1]), lo, n)

    def find_band_group(T):
        # the kernel's 32-way warp search for the first g with hi_g + C (g + 1) >= T
        key = lambda g: hi_of(g) + C * (g + 1)
        lo, cnt = 0, G
        while cnt > 32:
            step = (cnt + 31) // 32
            hits = [key(min(lo + (l + 1) * step - 1, lo + cnt - 1)) >= T for l in range(32)]
            if not any(hits):
                return lo + cnt
            k = hits.index(True)
            nlo = lo + k * step
            cnt = min(lo + (k + 1) * step - 1, lo + cnt - 1) - nlo + 1
            lo = nlo
        hits = [l < cnt and key(lo + l) >= T for l in range(32)]
        return lo + hits.index(True) if any(hits) else lo + cnt

    def band_range(k):
        if offsets is None:
            tiles = (n + STAGE - 1) // STAGE
            t0 = 0 if k <= 0 else min(n, STAGE * (tiles * k // bands))
            t1 = n if k + 1 >= bands else min(n, STAGE * (tiles * (k + 1) // bands))
            return t0, t1, 0
        edges = []
        for kk in (k, k + 1):
            T = ctot * kk // bands
            g = find_band_group(T)
            t = T - C * G if g >= G else min(T - C * g, hi_of(g))
            edges.append((clamp(t, 0, n), g))
        t0 = 0 if k <= 0 else edges[0][0]
        t1 = n if k + 1 >= bands else edges[1][0]
        g0 = 0 if k <= 0 else min(edges[0][1], G)
        return t0, t1, g0

    def first_band(g, seg_lo):
        if offsets is None:
            return 0
        cost = seg_lo + C * g
        return max(0, min(bands - 1, ((cost + 1) * bands - 1) // ctot))

    def slot_of(k, slab, s):
        return (k * slabs + slab) * 2 + s

    def in_workspace(slot):
        return 0 <= slot and part_off + 4 * PART_FLOATS * (slot + 1) <= total and \
            flag_off + 8 * (slot * 4 + 4) <= part_off

    ranges = [band_range(k) for k in range(bands)]
    if strict and offsets is not None:
        starts = [r[0] for r in ranges] + [n]
        assert all(starts[i] <= starts[i + 1] for i in range(bands)), starts
        assert all(ranges[k][1] == starts[k + 1] for k in range(bands))

    writes, published, owned, sums = {}, {}, set(), []
    cover = np.zeros((slabs, n), np.int32) if n * slabs < 3e7 else None
    for b in range(sgroups * bands):
        band, sg = divmod(b, sgroups)
        bt0, bt1, gb = ranges[band]
        sl0, sl1 = slabs * sg // sgroups, slabs * (sg + 1) // sgroups
        pending = None
        for slab in range(sl0, sl1):
            t, g = bt0, gb
            while t < bt1:
                lo = hi = 0
                while g < G:
                    lo, hi = group_range(g)
                    if hi > t:
                        break
                    g += 1
                if g >= G or lo >= bt1:
                    break
                t = max(t, lo)
                t1 = min(hi, bt1)
                assert 0 <= t <= t1 <= n
                if t1 == t:
                    continue
                if cover is not None:
                    cover[slab, t:t1] += 1
                if lo >= bt0:
                    role = OWNED if hi <= bt1 else FIRST_BAND
                else:
                    role = LAST_BAND if hi <= bt1 else MIDDLE
                if role == OWNED:
                    assert not strict or (slab, g) not in owned
                    owned.add((slab, g))
                else:
                    slot = slot_of(band, slab, 1 if role == FIRST_BAND else 0)
                    assert in_workspace(slot)
                    assert not strict or slot not in writes, ("slot reused", slot)
                    writes[slot] = (slab, g, band)
                    if role != LAST_BAND:
                        published[slot] = (b, False)
                    else:
                        assert not strict or pending in (None, (g, lo))
                        pending = (g, lo)
                t = t1
        if bt0 >= bt1:  # a band without tokens publishes empty flags
            for slab in range(sl0, sl1):
                published.setdefault(slot_of(band, slab, 0), (b, True))
        if pending is not None:
            for slab in range(sl0, sl1):
                sums.append((b, pending[0], slab, pending[1], band))

    read = set()
    for b, g, slab, lo, band in sums:
        b0 = first_band(g, lo)
        assert not strict or b0 < band, (b0, band)
        for kk in range(b0, band):
            slot = slot_of(kk, slab, 1 if kk == b0 else 0)
            assert in_workspace(slot)
            if strict:
                assert slot in published, ("never published", slot, kk, b0, band)
                writer, empty = published[slot]
                assert writer < b, "a wait on a CTA with a higher block index"
                if not empty:
                    assert writes.get(slot) == (slab, g, kk), (slot, writes.get(slot), (slab, g, kk))
                    read.add(slot)
        if strict:
            own = slot_of(band, slab, 0)
            assert writes.get(own) == (slab, g, band)
            read.add(own)
            assert (slab, g) not in owned
    if strict:
        assert read == set(writes), (len(read), len(writes))
        if cover is not None:
            want = np.zeros(n, np.int32)
            if offsets is None:
                want[:] = 1
            else:
                for g in range(G):
                    lo, hi = group_range(g)
                    want[lo:hi] += 1
            assert (cover == want[None, :]).all()
    return slabs, sgroups, bands


@pytest.mark.parametrize("cap", [296, 320, 8, 2])
def test_band_split_of_the_five_layers(cap):
    for cfg in range(5):
        sh = synth.config_shapes(cfg)
        off = None
        if cfg == 4:
            c = synth.zipf_counts(32768, 64, 1.1)
            off = np.concatenate([[0], np.cumsum(c)])
        check(sh["n_tok"], sh["c_in"], off, cap)


def test_band_split_random_offsets():
    rng = np.random.default_rng(0)
    for _ in range(150):
        n = int(rng.integers(1, 6000))
        c_in = 16 * int(rng.integers(1, 80))
        cap = int(rng.choice([296, 320, 7, 64, 150]))
        off = None
        if rng.random() < 0.7:
            G = int(rng.integers(1, 90))
            off = np.sort(rng.integers(-5, n + 5, G + 1))
            if rng.random() < 0.5:
                off[0], off[-1] = 0, n
            if rng.random() < 0.3:  # a pile of empty groups at one offset
                off = np.sort(np.concatenate([off, np.repeat(off[len(off) // 2], int(rng.integers(1, 60)))]))
        check(n, c_in, off, cap)


def test_band_split_wide_layer_and_bad_offsets():
    assert check(300, 128 * 700, None, 296) == (700, 296, 1)
    rng = np.random.default_rng(1)
    for _ in range(150):
        n = int(rng.integers(1, 3000))
        c_in = 16 * int(rng.integers(1, 40))
        off = rng.integers(-50, n + 50, int(rng.integers(1, 40)) + 1)  # any order: bounds only
        check(n, c_in, off, int(rng.choice([296, 320, 7, 64])), strict=False)
