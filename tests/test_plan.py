"""The fit pass's launch plan (host code, no GPU): its invariants, and an
emulation of the work distribution the pass runs over it.

The pass gives every warp a fixed first item (chunk gw / strips of strip
gw % strips, gw the warp's index in the grid); then each warp claims one item
at a time from its home strip's counter (counters start past the fixed
chunks), moving to the next strip when its own runs dry, until every strip is
dry or it holds max_items items.  Past 256 strips one counter hands out items
in order.  The emulation interleaves the warps at random and checks that
every (strip, row) is covered exactly once and no warp exceeds its item
bound, which is what keeps the fixed-point refine partials exact.
"""
import random

import pytest

from activation_aware_codebook_b200 import binding as bb
from activation_aware_codebook_b200.csrc import build as cbuild

WARPS_PER_BLOCK = 3
FULL_WAVE = 148 * 4
MAX_STRIPS = 256


@pytest.fixture(scope="module")
def lib():
    cbuild.build()
    return bb.load()


SHAPES = [(14336, 4096), (4096, 14336), (1024, 4096), (4096, 4096), (37, 640), (256, 512),
          (48, 257 * 512), (3, 128 * 1024), (27648, 5120), (1, 16), (8191, 4112)]


def weights_bound(M):
    # rows a warp may take: 2^(50 - B) / 16 with B = min(40, 61 - ceil(log2 M))
    c = 0
    while (1 << c) < M:
        c += 1
    B = min(40, 61 - c)
    return (1 << (50 - B)) // 16


@pytest.mark.parametrize("N,K", SHAPES)
@pytest.mark.parametrize("flags", [0, bb.CONCURRENT])
def test_plan_invariants(lib, N, K, flags):
    cfg = bb.Config(bb.INT4, 16, 16, 20, flags)
    p = bb.fit_launch_plan(cfg, N, K)
    strips = -(-K // 512)
    assert p["strips"] == strips
    assert p["items_per_strip"] == -(-N // p["item_rows"])
    items = strips * p["items_per_strip"]
    assert p["max_items"] == weights_bound(N * K) // p["item_rows"] >= 1
    warps = p["blocks"] * WARPS_PER_BLOCK
    # the warps' bounds cover every item, and no block is idle by construction
    assert warps * p["max_items"] >= items
    assert 1 <= p["blocks"] <= max(FULL_WAVE, -(-items // (WARPS_PER_BLOCK * p["max_items"])))
    assert p["blocks"] <= -(-items // WARPS_PER_BLOCK)  # at most one block per 3 items
    if flags & bb.CONCURRENT:
        full = bb.fit_launch_plan(bb.Config(bb.INT4, 16, 16, 20), N, K)
        share = max(16, -(-N * K // 196608))
        assert p["blocks"] == max(min(full["blocks"], share),
                                  -(-items // (WARPS_PER_BLOCK * p["max_items"])))


def test_sharded_plan_uses_the_whole_layer_for_the_bound(lib):
    cfg = bb.Config(bb.INT4, 128, 16, 20)
    whole = bb.fit_launch_plan(cfg, 14336, 4096)
    shard = bb.fit_launch_plan(cfg, 3584, 4096, N_total=14336)
    assert shard["max_items"] == whole["max_items"]
    assert shard["items_per_strip"] == -(-3584 // shard["item_rows"])


def test_plan_rejects_bad_arguments(lib):
    import ctypes
    out = (ctypes.c_int32 * 5)()
    c = bb.Config(bb.INT4, 128, 16, 20).c()
    assert lib.aaac_fit_launch_plan(ctypes.byref(c), 64, 256, 64, None) == 1
    assert lib.aaac_fit_launch_plan(None, 64, 256, 64, out) == 1
    assert lib.aaac_fit_launch_plan(ctypes.byref(c), 64, 200, 64, out) == 2   # K % g
    assert lib.aaac_fit_launch_plan(ctypes.byref(c), 64, 256, 32, out) == 2   # N_total < N
    assert lib.aaac_fit_launch_plan(ctypes.byref(c), 1 << 20, 4096, 1 << 20, out) == 2


def emulate(N, K, p, seed):
    """One round of the pass's work distribution over the plan p."""
    ncb, cpc, R, cap = p["strips"], p["items_per_strip"], p["item_rows"], p["max_items"]
    n_items = ncb * cpc
    wt = p["blocks"] * WARPS_PER_BLOCK
    per_strip = ncb <= MAX_STRIPS
    strip_next = [min(-(-(wt - i) // ncb), cpc) if i < ncb and i < wt else 0
                  for i in range(ncb)]
    next_item = [min(wt, n_items)]
    warps = []
    for gw in range(wt):
        first = None
        if per_strip:
            if gw // ncb < cpc:
                first = (gw % ncb, gw // ncb)
        elif gw < n_items:
            first = (gw // cpc, gw % cpc)
        warps.append(dict(cur=gw % ncb, tried=0, claimed=1 if first else 0,
                          items=[first] if first else [], done=first is None))
    covered = {}

    def claim(w):
        """One claim and its landing (a dry strip moves the warp on)."""
        while True:
            if w["done"] or w["claimed"] >= cap:
                w["done"] = True
                return
            w["claimed"] += 1
            if not per_strip:
                v = next_item[0]
                next_item[0] += 1
                if v < n_items:
                    w["items"].append((v // cpc, v % cpc))
                else:
                    w["claimed"] -= 1
                    w["done"] = True
                return
            v = strip_next[w["cur"]]
            strip_next[w["cur"]] += 1
            if v < cpc:
                w["items"].append((w["cur"], v))
                return
            w["claimed"] -= 1
            w["tried"] += 1
            if w["tried"] >= ncb:
                w["done"] = True
                return
            w["cur"] = (w["cur"] + 1) % ncb

    rng = random.Random(seed)
    live = [i for i, w in enumerate(warps) if not w["done"] or w["items"]]
    while live:
        i = rng.choice(live)
        w = warps[i]
        if w["items"]:
            strip, chunk = w["items"].pop(0)
            for r in range(chunk * R, min(N, chunk * R + R)):
                covered[(strip, r)] = covered.get((strip, r), 0) + 1
            if not w["items"]:
                claim(w)
        if not w["items"] and w["done"]:
            live.remove(i)
    assert all(w["claimed"] <= cap for w in warps)
    return covered


@pytest.mark.parametrize("N,K", [(1024, 4096), (37, 640), (48, 257 * 512), (300, 8192),
                                 (4096, 4096)])
@pytest.mark.parametrize("flags", [0, bb.CONCURRENT])
def test_work_distribution_covers_every_row_once(lib, N, K, flags):
    p = bb.fit_launch_plan(bb.Config(bb.INT4, 128, 16, 20, flags), N, K)
    for seed in range(3):
        covered = emulate(N, K, p, seed)
        assert len(covered) == p["strips"] * N
        assert set(covered.values()) == {1}


def emulate_ring(N, K, p, seed, stages=2):
    """The pass's per-warp producer/consumer over the plan p: a FIFO of
    items (8 entries) that the row prefetch fills as it crosses item ends, a
    ring of `stages` rows, and the consumer behind it.  Returns the rows each
    warp consumed, in order, and the deepest FIFO seen."""
    ncb, cpc, R, cap = p["strips"], p["items_per_strip"], p["item_rows"], p["max_items"]
    n_items = ncb * cpc
    wt = p["blocks"] * WARPS_PER_BLOCK
    per_strip = ncb <= MAX_STRIPS
    strip_next = [min(-(-(wt - i) // ncb), cpc) if i < ncb and i < wt else 0
                  for i in range(ncb)]
    next_item = [min(wt, n_items)]
    warps = []
    for gw in range(wt):
        first = -1
        fc = 0
        if per_strip:
            if gw // ncb < cpc:
                first, fc = gw % ncb, gw // ncb
        elif gw < n_items:
            first, fc = gw // cpc, gw % cpc
        w = dict(cur=gw % ncb, tried=0, claimed=1 if first >= 0 else 0, no_more=first < 0,
                 pend=None, pend_ok=False, fifo=[None] * 8, tail=1, pq=0, cq=0, ring=[],
                 rows=[], first=(first, fc))
        w["fifo"][0] = (first, fc)
        warps.append(w)

    def claim(w):
        w["pend_ok"] = (not w["no_more"]) and w["claimed"] < cap
        if w["pend_ok"]:
            if per_strip:
                w["pend"] = strip_next[w["cur"]]
                strip_next[w["cur"]] += 1
            else:
                w["pend"] = next_item[0]
                next_item[0] += 1
            w["claimed"] += 1

    def land_push(w):
        it, itc = -1, 0
        while w["pend_ok"]:
            v = w["pend"]
            if not per_strip:
                if v < n_items:
                    it, itc = v // cpc, v % cpc
                break
            if v < cpc:
                it, itc = w["cur"], v
                break
            w["claimed"] -= 1
            w["tried"] += 1
            if w["tried"] >= ncb:
                break
            w["cur"] = (w["cur"] + 1) % ncb
            claim(w)
        if it < 0:
            w["no_more"] = True
        assert w["tail"] - w["cq"] < 8, "FIFO overrun"
        w["fifo"][w["tail"] % 8] = (it, itc)
        w["tail"] += 1
        claim(w)

    def enter(w, ent):
        if ent[0] >= 0:
            w["pit"], w["pr"] = ent[0], ent[1] * R
            w["pe"] = min(N, w["pr"] + R)

    def prefetch(w):
        if w["fifo"][w["pq"] % 8][0] >= 0:
            w["ring"].append((w["pit"], w["pr"]))
            w["pr"] += 1
            if w["pr"] >= w["pe"]:
                w["pq"] += 1
                if w["pq"] == w["tail"]:
                    land_push(w)
                enter(w, w["fifo"][w["pq"] % 8])
        else:
            w["ring"].append(None)

    depth = 0
    for w in warps:  # prologue, first part: rows of the fixed item that do not end it
        w["pit"], w["pr"], w["pe"] = 0, 0, 0
        enter(w, w["first"])
        w["cit"], w["cr"], w["ce"] = (w["first"][0], w["pr"], w["pe"])
        w["npre"] = 0
        for k in range(stages):
            if w["first"][0] >= 0 and w["npre"] == k and w["pr"] + 1 < w["pe"]:
                w["ring"].append((w["pit"], w["pr"]))
                w["pr"] += 1
                w["npre"] += 1
    rng = random.Random(seed)
    order = list(range(wt))
    rng.shuffle(order)
    for i in order:  # after the dependency wait: one claim, then the rest of the ring
        claim(warps[i])
        for k in range(stages):
            if k >= warps[i]["npre"]:
                prefetch(warps[i])
    live = list(range(wt))
    while live:
        i = rng.choice(live)
        w = warps[i]
        if w["fifo"][w["cq"] % 8][0] < 0:
            live.remove(i)
            continue
        row = (w["cit"], w["cr"])
        w["cr"] += 1
        if w["cr"] >= w["ce"]:
            w["cq"] += 1
            e = w["fifo"][w["cq"] % 8]
            assert e is not None and w["cq"] < w["tail"], "consumer ahead of the FIFO"
            if e[0] >= 0:
                w["cit"], w["cr"], w["ce"] = e[0], e[1] * R, min(N, e[1] * R + R)
        assert w["ring"].pop(0) == row, "the ring slot holds another row"
        w["rows"].append(row)
        prefetch(w)
        depth = max(depth, w["tail"] - w["cq"])
    return [w["rows"] for w in warps], depth


@pytest.mark.parametrize("N,K", [(1024, 4096), (37, 640), (48, 257 * 512), (301, 8192),
                                 (4096, 4096), (7, 1024)])
@pytest.mark.parametrize("flags", [0, bb.CONCURRENT])
def test_ring_and_fifo(lib, N, K, flags):
    """Every row is prefetched into the ring before it is consumed, in the
    consumer's order; the FIFO never holds more than a few items; every row
    of every strip is consumed once."""
    p = bb.fit_launch_plan(bb.Config(bb.INT4, 128, 16, 20, flags), N, K)
    for seed in range(2):
        rows, depth = emulate_ring(N, K, p, seed)
        seen = [r for w in rows for r in w]
        assert len(seen) == len(set(seen)) == p["strips"] * N
        assert depth <= 3
