"""The prefill kernel's key-visibility rules (mask_rules.cuh, compiled for the
host) against the oracle's definitions: every bit of every 32-key word equals
key_allowed(query position, key position) for the position the slot or chunk
row holds (slot_positions for the caches, len + row for the chunk)."""
import os
import subprocess
import tempfile

import numpy as np

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "mixed_head_kv_b200", "csrc")


def test_mask_rules_match_the_key_sets():
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "mask_rules_check")
        subprocess.check_call(["g++", "-O1", "-std=c++17", "-I", CSRC, os.path.join(HERE, "mask_rules_check.cpp"),
                               "-o", exe])
        lines = subprocess.check_output([exe], text=True).splitlines()
    assert len(lines) > 10000
    slots = {}
    checked = 0
    for line in lines:
        src, retr, S, R, L, C, q, base, bits = (int(x) for x in line.split())
        pq = L + q
        for k in range(32):
            key = base + k
            if src == 0:
                want = key < L and oracle.key_allowed(1, pq, key, S, R)
            elif src == 1:
                if (S, R, L) not in slots:
                    slots[(S, R, L)] = oracle.slot_positions(0, S, R, L, S + R)
                pos = slots[(S, R, L)][key] if key < S + R else -1
                want = pos >= 0 and oracle.key_allowed(0, pq, int(pos), S, R)
            else:
                want = key < C and oracle.key_allowed(retr, pq, L + key, S, R)
            got = (bits >> k) & 1
            assert got == int(want), f"src {src} retr {retr} S {S} R {R} L {L} C {C} row {q} key {key}: {got}"
            checked += 1
    assert checked > 300000
