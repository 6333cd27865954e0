"""Host-side logic of the tile schedule shared by the three kernels
(gla_common.cuh: WorkPlan, TileCursor), tested on the real C++ compiled for
the host: every tile of every unit is visited exactly once, segments are
marked correctly, each (unit, CTA) segment gets a unique partial slot below
units + CTAs, and the scan's slot lookup names exactly the CTAs that wrote a
partial of each unit."""

import os
import subprocess
from collections import defaultdict

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "gated_linear_attention_frame_b200", "csrc")


@pytest.fixture(scope="module")
def plan_dump(tmp_path_factory):
    from gated_linear_attention_frame_b200.build import nvcc_path

    exe = str(tmp_path_factory.mktemp("plan") / "plan_dump")
    src = os.path.join(ROOT, "tests", "cpp", "plan_dump.cu")
    subprocess.run([nvcc_path(), "-std=c++17", "-O1", "-I", CSRC, src, "-o", exe], check=True,
                   capture_output=True)
    return exe


CASES = [
    # units, tiles per unit, CTAs   (720p-5s, 480p-5s, 720p-60s, stream, small shapes)
    (1008, 29, 148), (840, 13, 148), (5784, 29, 148), (192, 29, 148), (8, 1, 8),
    (2, 1, 2), (7, 3, 5), (1, 1, 1), (3, 40, 120), (1000, 1, 148), (148, 2, 148),
    (296, 5, 148), (149, 7, 148), (12, 8, 96),
]


@pytest.mark.parametrize("units,tpu,G", CASES)
def test_schedule(plan_dump, units, tpu, G):
    G = min(G, units * tpu)
    out = subprocess.run([plan_dump, str(units), str(tpu), str(G)], check=True,
                         capture_output=True, text=True).stdout.split("\n")
    tiles = defaultdict(list)        # unit -> tiles seen
    writers = defaultdict(set)       # unit -> CTAs that end a segment of it
    slots = {}
    per_cta = defaultdict(list)
    urange = {}
    for line in out:
        if not line:
            continue
        f = line.split()
        if f[0] == "T":
            c, u, t, first, last, slot = map(int, f[1:])
            per_cta[c].append((u, t, first, last, slot))
            tiles[u].append(t)
        else:
            u, c0, c1, s0 = map(int, f[1:])
            urange[u] = (c0, c1, s0)
    # every tile exactly once
    assert set(tiles) == set(range(units))
    for u, ts in tiles.items():
        assert sorted(ts) == list(range(tpu))
    assert len(per_cta) == G and all(per_cta[c] for c in range(G))  # no idle CTA
    for c, seq in per_cta.items():
        for k, (u, t, first, last, slot) in enumerate(seq):
            prev = seq[k - 1] if k else None
            nxt = seq[k + 1] if k + 1 < len(seq) else None
            assert first == int(prev is None or prev[0] != u)
            assert last == int(nxt is None or nxt[0] != u)
            if prev is not None and prev[0] == u:
                assert t == prev[1] + 1       # consecutive tiles inside a segment
            if last:
                assert slot not in slots, "slot reused"
                slots[slot] = (u, c)
                writers[u].add(c)
                assert 0 <= slot < units + G
    # the scan reads exactly the partials that were written
    for u in range(units):
        c0, c1, s0 = urange[u]
        expect = sorted(s for s, (uu, _) in slots.items() if uu == u)
        got = [s0 + k for k in range(c1 - c0 + 1)]
        assert got == expect, (u, got, expect)
    # full rounds: CTA c holds unit r*G + c whole
    rounds = units // G
    for c in range(G):
        for r in range(rounds):
            seg = [x for x in per_cta[c] if x[0] == r * G + c]
            assert len(seg) == tpu
