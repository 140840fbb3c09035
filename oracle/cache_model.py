"""Evict-oldest simulation of the two DuoAttention cache kinds, for tiny inputs.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py). Pure-Python loops.

A retrieval head's cache keeps every token. A streaming head's cache has
constant length: it keeps the attention-sink tokens (the first `sink`
positions, never evicted) and the `recent` most recent other tokens, evicting
the oldest non-sink token when a new one arrives (DuoAttention abstract;
project card "How It Works"). Tokens are appended before the new token's query
attends, so the query's own token is one of the `recent` tokens.

The ring-slot placement (slot = sink + (p - sink) mod recent) is this
library's layout choice, not something the pages fix; `ring_slots` simulates
it by writing each token into its slot in arrival order.
"""
from __future__ import annotations

from collections import deque
from typing import Dict, List


def retained_positions(is_retrieval: bool, sink: int, recent: int, length: int) -> List[int]:
    """Positions held by one head's cache after `length` tokens were appended."""
    sinks: List[int] = []
    window: deque = deque()
    for p in range(length):
        if is_retrieval:
            sinks.append(p)
            continue
        if len(sinks) < sink:
            sinks.append(p)
            continue
        window.append(p)
        if len(window) > recent:
            window.popleft()
    return sorted(sinks + list(window))


def ring_slots(sink: int, recent: int, length: int) -> Dict[int, int]:
    """slot -> position after appending tokens 0..length-1 one at a time into a
    fixed sink region plus a ring of `recent` slots."""
    slots: Dict[int, int] = {}
    nxt = 0  # next ring slot to overwrite
    for p in range(length):
        if p < sink:
            slots[p] = p
        else:
            slots[sink + nxt] = p
            nxt = (nxt + 1) % recent
    return slots
