"""Bookkeeping of the mask parity band.

Mask parity excuses a GPU/oracle mismatch only for pairs the oracle flags as
ambiguous (a threshold within 1e-6 of the prefixes near-equal masses allow,
or a cosine within 1e-6 of the gate).  ``check_band`` bounds how many pairs
a test may flag, so that a band gone wrong cannot make mask parity pass
without comparing anything, and records the counts; the pytest session
prints them at the end (tests/conftest.py)."""
from __future__ import annotations

COUNTS = []          # (test label, flagged pairs, compared pairs)
NOTES = []           # free-form lines printed at the end of the session (measured error ratios)
MAX_FRACTION = 1e-3


def check_band(label: str, n_flagged: int, n_pairs: int, max_fraction: float = MAX_FRACTION):
    COUNTS.append((label, int(n_flagged), int(n_pairs)))
    assert n_pairs > 0, label
    assert n_flagged <= max_fraction * n_pairs, \
        "%s: %d of %d pairs in the ambiguity band (> %.2g)" % (label, n_flagged, n_pairs, max_fraction)


def note(line: str):
    NOTES.append(line)
