"""The stream-K schedule's invariants, host arithmetic only (no GPU): for the
plans fp8_mm_plan returns with a workspace, the work items the kernel derives
(whole tiles round robin, then contiguous k-block ranges per CTA) cover every
k-block of every tile exactly once, every CTA writes at most one partial, a
cut tile's owner -- the CTA holding its first k-block -- has between one and
six partials (what its epilogue warps can stage in the operand ring), held by
exactly the CTAs after it, and every partial slot lies in the workspace.

The kernel's item rule, restated: range c = [c U / P, (c + 1) U / P) of the U
stream-K k-blocks (tiles in order, problem 0 first); a range's piece of a tile
starting at k-block 0 is that tile's owner part, a piece starting later is a
partial part; a tile's owner adds the partials of CTAs owner + 1 ..
cta_of(last k-block of the tile), where cta_of(u) = ceil((u + 1) P / U) - 1."""
import itertools

import pytest

A = 0x100000
WS = 0x8000000
SK = 8
MAX_PARTS = 6


@pytest.fixture(scope="module")
def fp8():
    import fp8_delayed_scaling_03_b200 as m
    return m


def mm_args(F, m, n, k, a_major, b_major, cfg, ws_bytes):
    lda = k if a_major == 0 else m
    ldb = k if b_major == 0 else n
    lda, ldb = (lda + 15) // 16 * 16, (ldb + 15) // 16 * 16
    a = F.MmArgs(m, n, k, A, 0, a_major, lda, A + 0x10000, 0, b_major, ldb, A + 0x20000, A + 0x20010,
                 None, 0, None, A + 0x30000, n, cfg)
    a.workspace, a.workspace_bytes = WS, ws_bytes
    return a


def simulate(tiles, kbs, units, D, P):
    """Items per CTA from the kernel's rule.  tiles: per-problem tile counts,
    kbs: per-problem k-blocks; units: the grid's CTAs (pairs) for the
    whole-tile round robin; D: whole tiles; P: stream-K CTAs."""
    T0 = tiles[0]
    total = sum(tiles)
    kb_of = lambda t: kbs[0] if t < T0 else kbs[1]  # noqa: E731
    u0 = (T0 - D) * kbs[0] if D < T0 else 0
    U = u0 + (total - max(D, T0)) * kbs[1]
    items = {c: [] for c in range(max(units, P))}
    for c in range(units):
        for t in range(c, D, units):
            items[c].append((t, 0, kb_of(t), "full", 0))

    def tile_of(u):
        if u < u0:
            t = D + u // kbs[0]
            return t, (t - D) * kbs[0]
        t1 = max(D, T0)
        t = t1 + (u - u0) // kbs[1]
        return t, u0 + (t - t1) * kbs[1]

    cta_of = lambda u: ((u + 1) * P + U - 1) // U - 1  # noqa: E731
    for c in range(P):
        u, ue = c * U // P, (c + 1) * U // P
        while u < ue:
            t, ut = tile_of(u)
            kb = u - ut
            take = min(kb_of(t) - kb, ue - u)
            if kb > 0:
                kind, nparts = "partial", 0
            elif take == kb_of(t):
                kind, nparts = "full", 0
            else:
                kind, nparts = "owner", cta_of(ut + kb_of(t) - 1) - c
            items[c].append((t, kb, kb + take, kind, nparts))
            u += take
    return items, total, kb_of


CASES = [
    (512, 1536, 1536, 0, 0), (512, 1536, 6912, 0, 1), (512, 6912, 1536, 1, 1), (2048, 1536, 1536, 0, 0),
    (2048, 1536, 6912, 0, 1), (2048, 6912, 1536, 0, 0), (1536, 6912, 2048, 1, 1), (4096, 4096, 4096, 0, 0),
    (4096, 11008, 4096, 0, 0), (4096, 4096, 11008, 0, 1), (3, 100, 1100, 0, 0), (300, 200, 1000, 1, 0),
    (64, 192, 640, 0, 1), (256, 384, 2048, 1, 1), (4096, 4096, 384, 0, 0), (700, 520, 3000, 0, 1),
]


@pytest.mark.parametrize("cfg", (1, 2, 3))
@pytest.mark.parametrize("m,n,k,a_major,b_major", CASES)
def test_schedule_covers_and_bounds_partials(fp8, m, n, k, a_major, b_major, cfg):
    F = fp8
    ws = F.fp8_mm_workspace_bytes(m, n, k)
    plan = F.fp8_mm_plan(mm_args(F, m, n, k, a_major, b_major, cfg | SK, ws), None, 148)
    assert plan.stream_k_ctas > 0
    tm, tn = (256, 256) if cfg == 3 else (128, 128 if cfg == 1 else 256)
    tiles = [((m + tm - 1) // tm) * ((n + tn - 1) // tn), 0]
    kbs = [(k + 127) // 128, 1]
    P = plan.stream_k_ctas
    D = plan.dp_tiles
    units = plan.units
    assert D % units == 0 if D else True
    items, total, kb_of = simulate(tiles, kbs, units, D, P)
    # every k-block of every tile exactly once
    seen = {}
    for c, its in items.items():
        for (t, lo, hi, kind, nparts) in its:
            for kb in range(lo, hi):
                assert (t, kb) not in seen, (t, kb)
                seen[(t, kb)] = c
    assert len(seen) == sum(kb_of(t) for t in range(total))
    slots = (ws - 160 * 8 * 4) // (128 * 256 * 4)
    per_unit = 2 if cfg == 3 else 1
    for c, its in items.items():
        kinds = [it[3] for it in its]
        assert kinds.count("partial") <= 1                      # one partial slot per CTA
        if "partial" in kinds:
            sk_items = [it for it in its if it[0] >= D]
            assert sk_items[0][3] == "partial"                  # the partial part comes first
            assert (c + 1) * per_unit <= slots                  # the slot lies in the workspace
        if "owner" in kinds:
            assert kinds[-1] == "owner"                         # the owner part comes last
        for (t, lo, hi, kind, nparts) in its:
            if kind != "owner":
                continue
            assert 1 <= nparts <= MAX_PARTS
            holders = sorted({seen[(t, kb)] for kb in range(hi, kb_of(t))})
            assert holders == list(range(c + 1, c + 1 + nparts))
            for h in holders:                                   # each holder's piece of t is its partial
                assert [it for it in items[h] if it[0] == t][0][3] == "partial"


def test_schedule_two_problems(fp8):
    """A dX + dW launch (unequal k) with forced stream-K on 128x256 tiles."""
    F = fp8
    M, N, K = 2100, 520, 300
    dx = mm_args(F, M, K, N, 0, 1, 2 | SK, F.fp8_mm_workspace_bytes(M, K, N))
    dw = mm_args(F, N, K, M, 1, 1, 2 | SK, 0)
    plan = F.fp8_mm_plan(dx, dw, 148)
    assert plan.stream_k_ctas > 0
    tiles = [((M + 127) // 128) * ((K + 255) // 256), ((N + 127) // 128) * ((K + 255) // 256)]
    kbs = [(N + 127) // 128, (M + 127) // 128]
    items, total, kb_of = simulate(tiles, kbs, plan.units, plan.dp_tiles, plan.stream_k_ctas)
    covered = sorted((t, kb) for its in items.values() for (t, lo, hi, _, _) in its for kb in range(lo, hi))
    assert covered == sorted((t, kb) for t in range(total) for kb in range(kb_of(t)))
    assert all(1 <= n_ <= MAX_PARTS for its in items.values() for (_, _, _, kind, n_) in its if kind == "owner")
