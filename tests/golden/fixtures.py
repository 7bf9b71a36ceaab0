"""Parser for the hand-worked text fixtures in this directory.

Each fixture file is a list of blocks separated by blank lines.  A block line
is ``key: values``; ``|`` separates matrix rows; numbers may be decimal or C99
hex floats.  Lines starting with ``#`` are comments.  Keys that appear before
the first case-specific key (a header block) are shared by later blocks.
"""
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def _num(tok):
    tok = tok.strip()
    if "0x" in tok.lower() or "p" in tok.lower():
        return float.fromhex(tok)
    return float(tok)


def _parse_value(text):
    rows = [r.split() for r in text.split("|")]
    if len(rows) == 1:
        return np.array([_num(t) for t in rows[0]], dtype=np.float64)
    return np.array([[_num(t) for t in r] for r in rows], dtype=np.float64)


def load_blocks(name):
    path = os.path.join(HERE, name)
    blocks, cur = [], {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            line = line.rstrip("\n")
            if line.startswith("#"):
                continue
            if not line.strip():
                if cur:
                    blocks.append(cur)
                    cur = {}
                continue
            key, val = line.split(":", 1)
            cur[key.strip()] = _parse_value(val)
    if cur:
        blocks.append(cur)
    return blocks
