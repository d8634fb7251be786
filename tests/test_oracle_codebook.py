"""Pins of the oracle's NF4 codebook and inverse normal CDF.

The printed table ("QLoRA: Mathematical Foundations ...", section "4-Bit
NormalFloat (NF4)") is the canonical codebook; the quantile construction of
the same section, with the outermost probability read as
delta = 1 - (1/30 + 1/32) / 2, must reproduce it within 1e-6.
"""
import math

import numpy as np
import pytest
from scipy.special import ndtri

from conftest import read_golden_values

DELTA = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)


def printed_levels():
    return [float(s) for s in read_golden_values("nf4_levels_printed.txt")]


def test_printed_values_are_exact_binary32():
    for v in printed_levels():
        assert float(np.float32(v)) == v


def test_oracle_table_equals_printed(oracle_mod):
    q = oracle_mod.codebook()
    assert q.dtype == np.float32
    assert [float(v) for v in q] == printed_levels()


def test_table_structure(oracle_mod):
    q = oracle_mod.codebook().astype(np.float64)
    assert q[0] == -1.0 and q[15] == 1.0 and q[7] == 0.0
    assert np.all(np.diff(q) > 0)
    assert int(np.sum(q < 0)) == 7 and int(np.sum(q > 0)) == 8


def test_norm_ppf_matches_library_routine(oracle_mod):
    ps = np.concatenate([np.linspace(1e-6, 1 - 1e-6, 401), [0.5, 0.025, 0.975, DELTA, 1 - DELTA]])
    for p in ps:
        assert abs(oracle_mod.norm_ppf(p) - float(ndtri(p))) < 1e-12


def test_norm_ppf_closed_forms(oracle_mod):
    assert abs(oracle_mod.norm_ppf(0.5)) < 1e-15
    # Phi(1) = (1 + erf(1/sqrt 2)) / 2
    assert abs(oracle_mod.norm_ppf(0.5 * (1 + math.erf(1 / math.sqrt(2)))) - 1.0) < 1e-12
    for p in (0.01, 0.2, 0.4):
        assert abs(oracle_mod.norm_ppf(p) + oracle_mod.norm_ppf(1 - p)) < 1e-12


def test_construction_reproduces_printed_table(oracle_mod):
    c = oracle_mod.codebook_construct(DELTA)
    pr = np.array(printed_levels())
    assert np.max(np.abs(c - pr)) <= 1e-6
    assert c[7] == 0.0 and c[0] == -1.0 and c[15] == 1.0
    assert np.all(np.diff(c) > 0)


def test_construction_detects_wrong_split(oracle_mod):
    """A symmetric 8/8 split or a wrong tail probability misses the table."""
    pr = np.array(printed_levels())
    far = oracle_mod.codebook_construct(0.99)
    assert np.max(np.abs(far - pr)) > 1e-3
    # mirror image (7 positive, 8 negative) is far from the printed table
    mirrored = -oracle_mod.codebook_construct(DELTA)[::-1]
    assert np.max(np.abs(mirrored - pr)) > 1e-2
