"""The debug-check build and the schedule checker.

The debug build (libe4b_debug.so, compiled with E4B_DEBUG_CHECKS=1) checks on the
device every m-tile entry and pair id the grouped GEMMs use, the row gather's pair
ids, the inverse-permutation entries of the combine and of the routing gradient,
and, after every grouping, the whole schedule.  A failed check records its site in
the status word and skips the access it guards; nothing traps.  This stands in for
a memory checker behind the expert-layer pages' "fails loudly" contract
(bitsandbytes PR #1965, "Correctness & coverage").

On valid inputs, dropped pairs included, the debug build must find nothing and
give the release build's results bit for bit (both run the same scenario in child
processes).  The schedule checker runs in both builds: fed a schedule built here
on the host from the routing, it must pass it, and once one field is corrupted it
must report the property that field breaks."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from bit_quantized_mixture_nf4_b200 import build as e4b_build

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TILE = 256


@pytest.fixture(scope="module")
def e4b():
    import bit_quantized_mixture_nf4_b200 as m
    m.lib
    return m


def _run(tmp_path, debug):
    e4b_build.build(debug=debug)
    out = os.path.join(tmp_path, f"run_{int(debug)}.npz")
    env = dict(os.environ, E4B_DEBUG="1" if debug else "0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_debug_run.py"), out], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    return dict(np.load(out))


def test_debug_build_finds_nothing_and_matches_release(tmp_path):
    rel = _run(str(tmp_path), False)
    dbg = _run(str(tmp_path), True)
    assert int(rel["debug_checks"]) == 0 and int(dbg["debug_checks"]) == 1
    for part in ("train", "given", "decode"):
        assert int(dbg[f"status_{part}"]) == 0, (part, hex(int(dbg.get(f"word_{part}", 0))))
        assert int(rel[f"status_{part}"]) == 0, part
    for k in ("y", "idx", "wts", "gx", "gw", "gl", "y2", "gx2", "yd"):
        assert np.array_equal(rel[k], dbg[k]), k


def host_schedule(idx, E, tile_rows, extra=4):
    """Grouping of the pairs by expert, stable in pair order, written from its
    definition: expert e owns the rows [offsets[e], offsets[e+1]); pairs naming an
    expert outside [0, E) are dropped (inv_perm -1)."""
    idx = idx.reshape(-1).astype(np.int64)
    P = idx.size
    valid = (idx >= 0) & (idx < E)
    order = np.argsort(np.where(valid, idx, E), kind="stable")
    counts = np.bincount(idx[valid], minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    n = int(offsets[-1])
    perm = np.zeros(P, np.int64)
    perm[:n] = order[:n]
    inv = -np.ones(P, np.int64)
    inv[order[:n]] = np.arange(n)
    tiles = (counts + tile_rows - 1) // tile_rows
    tile_prefix = np.concatenate([[0], np.cumsum(tiles)])
    sched = np.zeros((P // tile_rows + E + extra, 4), np.int64)
    m = 0
    for e in range(E):
        for j in range(tiles[e]):
            sched[m] = (e, offsets[e] + j * tile_rows, min(tile_rows, counts[e] - j * tile_rows), 0)
            m += 1
    return {"counts": counts, "offsets": offsets, "tile_prefix": tile_prefix, "sched": sched, "perm": perm,
            "inv_perm": inv}


def _validate(e4b, idx, E, s):
    dev = torch.device("cuda")
    t = {k: torch.from_numpy(np.ascontiguousarray(v).astype(np.int32)).to(dev) for k, v in s.items()}
    st = e4b.e4b_debug_validate_schedule(torch.from_numpy(idx.astype(np.int32)).to(dev), E, TILE, t["counts"],
                                         t["offsets"], t["tile_prefix"], t["sched"], t["perm"], t["inv_perm"])
    return st, (e4b.e4b_last_status_word() >> 8) & 0xFF


@pytest.fixture(scope="module")
def routing():
    rng = np.random.default_rng(7)
    T, k, E = 700, 4, 6
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    idx[::9, 2] = -1          # dropped pairs
    idx[5::13, 3] = E + 2
    return idx, E


def test_schedule_checker_passes_a_consistent_schedule(e4b, routing):
    idx, E = routing
    s = host_schedule(idx, E, TILE)
    assert _validate(e4b, idx, E, s) == (e4b.E4B_OK, 0)


def _corrupt(s, what):
    s = {k: v.copy() for k, v in s.items()}
    E = s["counts"].size
    if what == "counts":
        s["counts"][1] += 1
    elif what == "tile_prefix":
        s["tile_prefix"][E] -= 1
    elif what == "sched_row0":
        s["sched"][1, 1] += 1             # an m-tile that does not start on a tile boundary
    elif what == "sched_expert":
        s["sched"][0, 0] = E + 5
    elif what == "perm_expert":             # two rows of different experts swap their pairs
        r1, r2 = s["offsets"][0], s["offsets"][1]
        p1, p2 = s["perm"][r1], s["perm"][r2]
        s["perm"][r1], s["perm"][r2] = p2, p1
        s["inv_perm"][p1], s["inv_perm"][p2] = r2, r1
    elif what == "perm_range":
        s["perm"][3] = 10 ** 6               # the pair row 3 held still points at row 3
    elif what == "inv_perm":
        p = s["perm"][5]
        s["inv_perm"][p] = -1
    elif what == "offsets":
        s["offsets"][0] = 1
    return s


@pytest.mark.parametrize("what,sites", [
    ("counts", {7}), ("tile_prefix", {8}), ("sched_row0", {9}), ("sched_expert", {9}), ("perm_expert", {10}),
    ("perm_range", {10, 11}), ("inv_perm", {11}), ("offsets", {6, 7, 9, 10})])
def test_schedule_checker_names_the_broken_property(e4b, routing, what, sites):
    idx, E = routing
    st, site = _validate(e4b, idx, E, _corrupt(host_schedule(idx, E, TILE), what))
    assert st == e4b.E4B_ERR_DEBUG_CHECK
    assert site in sites, (what, site)
    assert e4b.e4b_device_status() == e4b.E4B_OK   # read and cleared
