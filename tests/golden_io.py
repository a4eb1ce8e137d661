"""Readers for the hand-worked fixtures in tests/golden/ (plain text)."""
import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            yield [p.strip() for p in line.split("|")]


def hexbytes(s):
    return bytes(int(b, 16) for b in s.split())
