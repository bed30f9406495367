"""Readers for the text fixtures under tests/golden/."""
from __future__ import annotations

import os
from typing import Dict, List

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_table(name: str) -> List[List[str]]:
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


def read_cases(name: str) -> Dict[str, Dict[str, str]]:
    """Sections "[name]" followed by "key: value" lines (indented lines continue a value)."""
    cases: Dict[str, Dict[str, str]] = {}
    cur = None
    key = None
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            if raw.startswith("#"):
                continue
            line = raw.rstrip("\n")
            if not line.strip():
                continue
            if line.startswith("["):
                cur = {}
                cases[line.strip()[1:-1]] = cur
                key = None
            elif line.startswith(" ") and key is not None:
                cur[key] += " " + line.strip()
            else:
                key, _, val = line.partition(":")
                key = key.strip()
                cur[key] = val.strip()
    return cases


def pairs(spec: str) -> Dict[int, float]:
    out = {}
    for tok in spec.split():
        i, v = tok.split(":")
        out[int(i)] = float(v)
    return out


def byte_pairs(spec: str) -> Dict[int, int]:
    out = {}
    for tok in spec.split():
        i, v = tok.split(":")
        out[int(i)] = int(v, 16)
    return out


def expand(spec: str, n: int, fill=0.0):
    vals = [fill] * n
    for i, v in pairs(spec).items():
        vals[i] = v
    return vals


def expand_bytes(spec: str, n: int) -> bytes:
    b = bytearray(n)
    for i, v in byte_pairs(spec).items():
        b[i] = v
    return bytes(b)
