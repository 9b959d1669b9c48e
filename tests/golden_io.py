"""Readers for the small text fixtures under tests/golden/ (values printed on the pages)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            s = raw.strip()
            if s and not s.startswith("#"):
                yield s


def floats(s):
    return [float(v) for v in s.split()]
