"""Readers for the small text fixtures in tests/golden/ (no arithmetic)."""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def _lines(name):
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def max1960():
    out = {"threshold": {}, "level": {}, "mse": None}
    for kind, idx, val in _lines("max1960_gauss_8level.txt"):
        if kind == "mse":
            out["mse"] = float(val)
        else:
            out[kind][int(idx)] = float(val)
    return out


def packing():
    return {parts[0]: [int(w, 16) for w in parts[1:]] for parts in _lines("packing_examples.txt")}
