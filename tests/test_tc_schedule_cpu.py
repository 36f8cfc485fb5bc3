"""The tensor-core kernel's work split (dg_tc_schedule, host only): every shape
the kernels accept is checked on the CPU for complete, non-overlapping coverage
of the two contractions, for partial-sum slots in range, and for progress of
the hand-off between the two roles (no circular wait).

The progress model follows the kernel's rules as include/dg.h states them:
G1 units take vocabulary tiles from one queue in tile order, each holding one
tile until its ring slot is free (every G2 consumer of the tile `ring` places
earlier has loaded it); G2 units take their ranges in order, each waiting until
the range's tiles are complete. Counters only grow, so if repeatedly letting
every enabled unit advance finishes the step, no interleaving can deadlock.
"""
import itertools

import pytest

import synthetic
import uniform_state_text_b200 as dg

BN = 256          # vocabulary entries per tile and per range
BM = 128          # rows per row block


def g2_units(s):
    """(group g, row blocks, column slice) of every G2 unit, as include/dg.h defines them."""
    RBI = 1 if s["CG"] == 2 else s["RB"]
    for o in range(s["n2"]):
        g = o // (RBI * s["n_dt"])
        rem = o % (RBI * s["n_dt"])
        rows = tuple(range(s["RB"])) if s["CG"] == 2 else (rem // s["n_dt"],)
        yield g, rows, rem % s["n_dt"]


def check_shape(C, V, d, sms=148):
    s = dg.dg_tc_schedule(C, V, d, sms)
    CG, W2, RB, G = s["CG"], s["W2"], s["RB"], s["G"]
    RBI = 1 if CG == 2 else RB
    # geometry
    assert s["ctas"] == CG * (s["n1"] + s["n2"]) <= sms
    assert RB * BM == C and s["n_vt"] == V // BN and s["n_ranges"] == V // BN
    assert s["n_dt"] * W2 * BN == d
    assert s["n2"] == RBI * s["n_dt"] * G and s["n1"] >= 1 and 1 <= G <= s["n_ranges"]
    assert CG in (1, 2) and W2 in (1, 2) and (W2 == 1 or CG == 2)
    # coverage of P.E: every (range, row block, slice) exactly once; partial slots unique
    cover, slots = set(), set()
    units = list(g2_units(s))
    for g, rows, dt in units:
        assert 0 <= g < G and 0 <= dt < s["n_dt"]
        for rb in rows:
            assert (g, rb, dt) not in slots
            slots.add((g, rb, dt))
            for r in range(g, s["n_ranges"], G):
                assert (r, rb, dt) not in cover
                cover.add((r, rb, dt))
    assert len(cover) == s["n_ranges"] * RB * s["n_dt"]
    # progress of the hand-off
    ring, n_vt = s["ring"], s["n_vt"]
    # every tile resident up to 128 tiles, else 72 (CTA pairs) or 84 (single CTAs)
    assert ring == (n_vt if n_vt <= 128 else min(n_vt, 72 if CG == 2 else 84))
    consumers = RBI * s["n_dt"]               # G2 units that load each tile
    ready = [0] * n_vt                        # row blocks of the tile written
    consumed = [0] * n_vt
    items = n_vt * RBI                        # G1 queue entries, in tile order
    nxt, held = 0, []
    pos = [0] * len(units)
    ranges = [list(range(g, s["n_ranges"], G)) for g, _, _ in units]
    moved = True
    while moved:
        moved = False
        while len(held) < s["n1"] and nxt < items:     # free G1 units take the next tiles
            held.append(nxt)
            nxt += 1
            moved = True
        for it in list(held):                           # a held tile completes once its slot is free
            vt = it // RBI
            if vt < ring or consumed[vt - ring] >= consumers:
                ready[vt] += RB if CG == 2 else 1
                held.remove(it)
                moved = True
        for u, rs in enumerate(ranges):                 # G2 units take their ranges in order
            while pos[u] < len(rs) and ready[rs[pos[u]]] >= RB:
                consumed[rs[pos[u]]] += 1
                pos[u] += 1
                moved = True
    assert nxt == items and not held, "G1 stalled"
    assert all(p == len(rs) for p, rs in zip(pos, ranges)), "G2 stalled"
    assert all(c == consumers for c in consumed)
    return s


WORKLOAD_SHAPES = sorted({(w.C, w.V, w.d) for w in synthetic.WORKLOADS.values()
                          if w.C in (128, 256) and w.dtype == synthetic.BF16})
GPU_TEST_SHAPES = [(128, 256, 256), (256, 512, 256), (128, 4096, 256), (256, 8192, 512),
                   (128, 16384, 768)]


@pytest.mark.parametrize("shape", WORKLOAD_SHAPES + GPU_TEST_SHAPES)
def test_schedule_of_tested_shapes(shape):
    check_shape(*shape)


def test_headline_split():
    s = check_shape(256, 262144, 2048)
    assert (s["CG"], s["W2"], s["G"], s["n1"], s["n2"], s["ctas"]) == (2, 2, 8, 42, 32, 148)


@pytest.mark.parametrize("C,V,d", list(itertools.product(
    (128, 256), (256, 768, 4096, 32768, 65536), (256, 512, 768, 1024, 2048, 2816, 4096, 8192))))
def test_schedule_grid(C, V, d):
    check_shape(C, V, d)


@pytest.mark.parametrize("sms", [132, 148, 160])
def test_schedule_other_gpu_sizes(sms):
    check_shape(256, 262144, 2048, sms)
    check_shape(128, 262144, 2816, sms)


def test_uncovered_shapes_are_rejected():
    for C, V, d in [(64, 4096, 256), (256, 4096, 200), (256, 100, 256), (192, 4096, 256)]:
        with pytest.raises(dg.DgError) as e:
            dg.dg_tc_schedule(C, V, d)
        assert e.value.code == dg.DG_EUNSUPPORTED
    with pytest.raises(dg.DgError) as e:
        dg.dg_tc_schedule(256, 4096, 256, sms=1)
    assert e.value.code == dg.DG_EINVAL
