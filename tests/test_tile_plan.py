"""The prefill launch's work items and key-tile lists (tile_plan.cuh, compiled
for the host) against the key-set definitions of the oracle (its dense mask and slot model):

- every (batch, query head, query tile) with chunk rows is an item, once;
- every key a query row of the item may see lies in a listed tile (cache keys
  in the tile of the slot that holds them, chunk keys in their chunk tile);
- no retrieval-cache or chunk tile is fully masked for every row of the item
  (such tiles are skipped, which is where the prefill saves work); streaming-
  cache tiles are listed for all held slots once the window of the item's
  first row reaches below len (a superset, never past the held slots); no tile
  is listed twice.
"""
import itertools
import os
import subprocess
import tempfile

import numpy as np

import oracle
from oracle import brute

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
T = 128


def _cases():
    out = []
    for S, R, L, C in itertools.product((0, 4, 64), (1, 64, 200), (0, 3, 70, 300, 700), (1, 130, 300)):
        out.append((1, 4, 2, S, R, C, False, [L], [C], [1, 0]))
    # GQA, two sequences, ragged lengths and chunks
    for S, R in ((4, 64), (64, 256), (0, 17)):
        out.append((2, 8, 4, S, R, 300, True, [650, 5], [300, 131], [0, 1, 1, 0]))
        out.append((2, 8, 4, S, R, 260, True, [0, 1000], [7, 260], [1, 0, 0, 1]))
    return out


def _plan(cases):
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "tile_plan_check")
        subprocess.check_call(["g++", "-O1", "-std=c++17", "-I", os.path.join(ROOT, "include"), "-I",
                               os.path.join(ROOT, "mixed_head_kv_b200", "csrc"), "-I", "/usr/local/cuda/include",
                               os.path.join(HERE, "tile_plan_check.cpp"), "-o", exe])
        lines = []
        for (B, Hq, Hkv, S, R, C, ragged, lens, cs, mask) in cases:
            if ragged:
                seq = " ".join(f"{l} {c}" for l, c in zip(lens, cs))
            else:
                seq = str(lens[0])
            lines.append(f"{B} {Hq} {Hkv} {S} {R} {C} {int(ragged)} {seq} {' '.join(map(str, mask))}")
        text = subprocess.check_output([exe], input="\n".join(lines) + "\n", text=True)
    blocks, cur = [], []
    for line in text.splitlines():
        if line == "end":
            blocks.append(cur)
            cur = []
        else:
            f = [int(x) for x in line.split()[1:]]
            b, head, qt, retr, L, C, n = f[:7]
            tiles = [(f[7 + 2 * i], f[8 + 2 * i]) for i in range(n)]
            cur.append((b, head, qt, retr, L, C, tiles))
    return blocks


def _visible_tiles(retr, L, C, q0, S, R, slot_pos):
    """Tiles holding at least one key visible to some row of the query tile, each
    row's visible keys (the oracle's dense mask) mapped to their tile."""
    last = min(q0 + T, C)
    mask = brute.head_mask(L + last, bool(retr), S, R)[L + q0:L + last]  # rows q0 .. last-1
    keys = np.nonzero(mask.any(axis=0))[0]
    need = set()
    for j in keys.tolist():
        if j >= L:
            need.add((2, ((j - L) // T) * T))
        elif retr:
            need.add((0, (j // T) * T))
        else:
            slot = int(np.nonzero(slot_pos == j)[0][0])  # the slot that holds position j
            need.add((1, (slot // T) * T))
    return need


def test_items_cover_every_visible_key_and_skip_masked_tiles():
    cases = _cases()
    plans = _plan(cases)
    assert len(plans) == len(cases)
    for (B, Hq, Hkv, S, R, C, ragged, lens, cs, mask), items in zip(cases, plans):
        G = Hq // Hkv
        seen = set()
        for (b, head, qt, retr, L, Cb, tiles) in items:
            assert L == lens[b if ragged else 0] and Cb == cs[b if ragged else 0]
            assert retr == mask[head // G]
            q0 = qt * T
            if q0 >= Cb:
                assert tiles == []  # a query tile past this sequence's chunk
                continue
            key = (b, head, qt)
            assert key not in seen
            seen.add(key)
            assert len(set(tiles)) == len(tiles), "a tile is listed twice"
            slot_pos = oracle.slot_positions(0, S, R, L, S + R)
            need = _visible_tiles(retr, L, Cb, q0, S, R, slot_pos)
            assert need <= set(tiles), f"case {(S, R, L, Cb)} item {key}: missing {need - set(tiles)}"
            extra = set(tiles) - need
            assert all(src == 1 for src, _ in extra), f"case {(S, R, L, Cb)} item {key}: fully masked {extra}"
            held = min(L, S + R)
            assert all(row0 < held for src, row0 in tiles if src == 1), "a streaming tile past the held slots"
        expected = {(b, h, qt) for b in range(B) for h in range(Hq)
                    for qt in range((cs[b if ragged else 0] + T - 1) // T)}
        assert seen == expected
