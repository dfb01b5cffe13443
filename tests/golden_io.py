"""Reader for the hand-derived fixtures under tests/golden (key: values lines)."""
from __future__ import annotations

import os

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _num(tok: str):
    if tok.lower().startswith("0x") or tok.lower().startswith("-0x"):
        return int(tok, 16)
    if tok.lower() in ("nan", "-nan"):
        return float("nan")
    try:
        return int(tok)
    except ValueError:
        return float(tok)


def load(name: str) -> dict:
    out = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, _, rest = line.partition(":")
            toks = rest.split()
            vals = [_num(t) if key not in ("fmt",) else t for t in toks]
            out[key.strip()] = vals if len(vals) != 1 else vals[0]
    return out
